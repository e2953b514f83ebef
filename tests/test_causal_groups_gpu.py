"""Launches in the library's L2-aware orders: causal heads in L2-sized
groups, or pairs of query blocks head by head (even and odd block counts,
a ragged tail); tile-mask rows one head after another.

Output and LSE start as NaN, so a (head, query block) item the schedule
failed to deal would stay NaN; sampled rows (first, middle and last query
blocks) of the first head, a middle one and one in the partial last group are
checked against the oracle.
"""

import numpy as np
import pytest
import torch

import precision_attention_nvfp4_b200 as fp
import workloads
import parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,fmt", [(4, 32, 4096, "nvfp4"), (16, 64, 2048, "nvfp4"), (8, 64, 1024, "nvfp4"),
                                        (4, 23, 6144, "fp8"), (10, 8, 12123, "nvfp4")])
def test_causal_schedule_covers_every_item(B, H, N, fmt):
    d = 128
    plan = fp.causal_plan(B * H, N, d, fmt, "fp8", sm_count=torch.cuda.get_device_properties(0).multi_processor_count)
    # the grouped or the paired order is the one under test
    assert plan["heads_per_group"] < B * H or plan["pairs_per_head"] > 0, plan
    w = workloads.Workload("t", B=B, H=H, N=N, d=d, causal=True, qk_format=fmt, seed=21)
    q, k, v = workloads.make_qkv(w)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    if fmt == "nvfp4":
        qq, kq = fp.quantize_nvfp4(qc), fp.quantize_nvfp4(kc)
    else:
        qq, kq = fp.quantize_fp8(qc, "tile128"), fp.quantize_fp8(kc, "tile128")
    vq = fp.quantize_fp8(vc, "channel")
    out = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    fp.attention_fwd(qq, kq, vq, causal=True, out=out, lse=lse)
    torch.cuda.synchronize()
    assert fp.device_error() == 0
    assert not torch.isnan(out).any().item()
    assert not torch.isnan(lse).any().item()
    G = plan["heads_per_group"]
    heads = [0, (B * H) // 2, (B * H // G) * G if (B * H) % G else B * H - 1]
    nblk = -(-N // 128)
    rows = np.concatenate([np.arange(b * 128, min(N, b * 128 + 128)) for b in (0, nblk // 2, nblk - 1)])
    o = out.float().cpu().numpy().reshape(B * H, N, d)
    ls = lse.cpu().numpy().reshape(B * H, N)
    qh, kh, vh = parity.oracle_operands(q, k, v, fmt, heads)
    for i, bh in enumerate(heads):
        res = parity.compare_attention(o[bh], ls[bh], qh[i], kh[i], vh[i], rows, causal=True)
        parity.assert_close(res, f"{fmt} B{B} H{H} N{N} head {bh}")


def test_tile_mask_heads_one_after_another_cover_every_row():
    """Tile-mask launches take one head's rows after another: with output and
    LSE starting as NaN, every row of every head must be written, and sampled
    rows of the first, a middle and the last head match the oracle."""
    from oracle import sta
    grid, tile, window = (12, 16, 24), (6, 8, 8), (3, 3, 5)
    B, H, N, d = 2, 5, 12 * 16 * 24, 128
    w = workloads.Workload("t", B=B, H=H, N=N, d=d, causal=False, qk_format="fp8", seed=23)
    q, k, v = workloads.make_qkv(w)
    tg = tuple(a // b for a, b in zip(grid, tile))
    mask = fp.sta_plan(tg, tile, window).to("cuda")
    qq, kq = fp.quantize_fp8(q.cuda(), "tile128"), fp.quantize_fp8(k.cuda(), "tile128")
    vq = fp.quantize_fp8(v.cuda(), "channel")
    out = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    fp.attention_fwd(qq, kq, vq, tile_mask=mask, out=out, lse=lse)
    torch.cuda.synchronize()
    assert fp.device_error() == 0
    assert not torch.isnan(out).any().item()
    assert not torch.isnan(lse).any().item()
    heads = [0, (B * H) // 2, B * H - 1]
    nblk = N // 128
    rows = np.concatenate([np.arange(b * 128, b * 128 + 128) for b in (0, nblk // 2, nblk - 1)])
    o = out.float().cpu().numpy().reshape(B * H, N, d)
    ls = lse.cpu().numpy().reshape(B * H, N)
    qh, kh, vh = parity.oracle_operands(q, k, v, "fp8", heads)
    kb = sta.block_lists(grid, tile, window)
    for i, bh in enumerate(heads):
        res = parity.compare_attention(o[bh], ls[bh], qh[i], kh[i], vh[i], rows, key_blocks=kb)
        parity.assert_close(res, f"sta head {bh}")
