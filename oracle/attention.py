"""fp64 attention with an online softmax over 128-key tiles: TEST INFRASTRUCTURE ONLY.

What is computed (per query row i of one (batch, head)):
  scaled dot-product attention softmax(q k^T / sqrt(d)) v
    (FP4-attention tutorial page, section 2.1; FlashAttention-4 article,
     "online softmax" and tiling),
  evaluated the way a fused FlashAttention kernel evaluates it: keys are
  walked in ascending 128-key tiles aligned to key 0, keeping a running row
  max m, a running row sum l and an output accumulator O. For each tile:
      S_j  = softmax_scale * (q_i . k_j)          for the allowed keys j
      m'   = max(m, max_j S_j)
      P_j  = exp(S_j - m')
      l    = l * exp(m - m') + sum_j P_j          (unquantized P)
      Ph_j = E4M3(448 * P_j) / 448                (P at the fixed 1/448 tensor
                                                   scale, FPSAttention page,
                                                   section 3.1)
      O    = O * exp(m - m') + sum_j Ph_j v_j
      m    = m'
  and finally out = O / l, lse = m + ln(l).
A tile with no allowed key leaves the state unchanged. A row with no allowed
key at all gives out = 0 and lse = -inf.

Conditional rescale (FlashAttention-4 article, co-design list, online-softmax
item: rescale only once the running max has moved past a threshold),
``rescale_threshold`` = tau >= 0 in log2 units. The reference max m moves only
when it must:
      m_c  = max(m, max_j S_j)
      m'   = m_c   if m = -inf or (m_c - m) * log2(e) > tau,   else m
and the rest of the step is unchanged, except that P_j = exp(S_j - m') may
now reach 2^tau, so P is rounded at the scale 448 * 2^-tau, which keeps every
code below the E4M3 maximum:
      Ph_j = E4M3(448 * 2^-tau * P_j) / (448 * 2^-tau).
tau = 0 is the exact running max above.

All-NVFP4 variant (``p_format="nvfp4"``): P is quantized with the NVFP4
recipe of oracle.quant (Blackwell FP4 page, section 1: blocks of 16 along the
keys of the tile, E4M3 block scales) with its tensor amax fixed at 2^tau, the
bound of P under the reference max. This is the 4-bit counterpart of the fixed
FP8 P scale; the pages give no P rule for FP4, so this is the reading:
      Ph_j = NVFP4(P_j; A_t = 2^tau)   (P widened to float32 first)
V is then quantized along the sequence (oracle.quant.quantize_nvfp4_tokens),
which only changes the dequantized v passed in.

Allowed keys: all keys < N; under ``causal`` only j <= i; under a tile mask
only keys whose 128-key block is listed for the query's 128-row block.

Reading taken where the pages are silent: the row sum l adds the unquantized
P (so each row of P/l sums to one); ``quantize_p=False`` gives plain fp64
attention (P kept exact), used to pin the oracle to a textbook softmax.

Inputs are the dequantized fp64 operands q, k, v of one (batch, head), shaped
[N, d]. The loop over query rows is vectorized over one 128-row block at a
time; each row's arithmetic is the sequence above, unchanged.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

from . import codec, quant

TILE = 128
P_SCALE_INV = 448.0
LOG2E = 1.0 / math.log(2.0)


def _quantize_p(p: np.ndarray, tau: float = 0.0, fmt: str = "e4m3") -> np.ndarray:
    if fmt == "nvfp4":
        R, K = p.shape
        Kp = -(-K // quant.NVFP4_BLOCK) * quant.NVFP4_BLOCK
        pp = np.zeros((R, Kp), dtype=np.float32)
        pp[:, :K] = p.astype(np.float32)
        codes, sb, s_t = quant.quantize_nvfp4(pp, static_amax=2.0 ** tau)
        return quant.dequantize_nvfp4(codes, sb, s_t)[:, :K]
    assert fmt == "e4m3"
    s = P_SCALE_INV * 2.0 ** -tau
    return codec.e4m3_decode(codec.e4m3_encode(p * s)) / s


def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, rows: np.ndarray,
                   *, softmax_scale: Optional[float] = None, causal: bool = False,
                   key_blocks: Optional[Sequence[Sequence[int]]] = None,
                   quantize_p: bool = True, rescale_threshold: float = 0.0, p_format: str = "e4m3"):
    """Attention output and lse for the query ``rows`` of one (batch, head).

    q, k, v     float64 [N, d] dequantized operands
    rows        int array of query indices (all in one 128-row block, or any)
    key_blocks  optional list: key_blocks[qb] = allowed 128-key block indices
                for query block qb (the tile mask); None = dense
    rescale_threshold  tau of the conditional rescale (log2 units), 0 = exact
    p_format    "e4m3" (fixed 1/448 scale) or "nvfp4" (see the module notes)
    Returns (out float64 [len(rows), d], lse float64 [len(rows)]).
    """
    tau = float(rescale_threshold)
    assert tau >= 0.0
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.int64)
    N, d = k.shape
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    R = len(rows)
    m = np.full(R, -np.inf)
    l = np.zeros(R)
    O = np.zeros((R, v.shape[1]))
    ntiles = -(-N // TILE)
    qblk = rows // TILE
    listed_sets = None
    if key_blocks is not None:
        listed_sets = {int(b): set(key_blocks[b]) for b in np.unique(qblk)}
    for t in range(ntiles):
        keys = np.arange(t * TILE, min((t + 1) * TILE, N))
        allowed = np.ones((R, len(keys)), dtype=bool)
        if causal:
            allowed &= keys[None, :] <= rows[:, None]
        if key_blocks is not None:
            listed = np.array([t in listed_sets[int(b)] for b in qblk])
            allowed &= listed[:, None]
        live = allowed.any(axis=1)
        if not live.any():
            continue
        S = softmax_scale * (q[rows] @ k[keys].T)
        S = np.where(allowed, S, -np.inf)
        m_cand = np.where(live, np.maximum(m, S.max(axis=1)), m)
        with np.errstate(invalid="ignore"):
            move = np.isneginf(m) | ((m_cand - m) * LOG2E > tau)
        m_new = np.where(move, m_cand, m)
        with np.errstate(invalid="ignore"):
            alpha = np.where(live, np.exp(m - m_new), 1.0)
            P = np.where(allowed, np.exp(S - m_new[:, None]), 0.0)
        l = l * alpha + P.sum(axis=1)
        Ph = _quantize_p(P, tau, p_format) if quantize_p else P
        O = O * alpha[:, None] + Ph @ v[keys]
        m = m_new
    with np.errstate(invalid="ignore", divide="ignore"):
        out = np.where(l[:, None] > 0, O / np.where(l > 0, l, 1.0)[:, None], 0.0)
        lse = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return out, lse


def attention(q, k, v, *, softmax_scale=None, causal=False, key_blocks=None,
              quantize_p=True, rescale_threshold=0.0, p_format="e4m3"):
    """Whole (batch, head) attention, 128 rows at a time. Returns (out, lse)."""
    N = q.shape[0]
    outs, lses = [], []
    for b0 in range(0, N, TILE):
        rows = np.arange(b0, min(b0 + TILE, N))
        o, s = attention_rows(q, k, v, rows, softmax_scale=softmax_scale, causal=causal,
                              key_blocks=key_blocks, quantize_p=quantize_p,
                              rescale_threshold=rescale_threshold, p_format=p_format)
        outs.append(o)
        lses.append(s)
    return np.concatenate(outs), np.concatenate(lses)

