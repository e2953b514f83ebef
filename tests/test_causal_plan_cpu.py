"""Causal schedule of the attention kernel (host logic, no GPU).

fpattn_causal_plan reports how a causal launch deals its (head, query block)
items to the persistent CTAs: heads in groups whose K/V fit a share of the
L2, each group padded to whole pairs of snake rounds. These tests walk the
schedule by the rules the header states and check that every item is dealt
exactly once, that the padding keeps the balance it promises, and that a
group's K/V bytes fit the share.
"""

import numpy as np
import pytest

import precision_attention_nvfp4_b200 as fp

L2_SHARE = 32 * 2**20


def _walk(plan, bh, n):
    """(cta, head, query block) of every position that holds an item."""
    nblk = -(-n // 128)
    C, G, span, total = plan["ctas"], plan["heads_per_group"], plan["group_positions"], plan["positions"]
    pos = np.arange(total)
    rnd, c = pos // C, pos % C
    cta = np.where(rnd % 2 == 1, C - 1 - c, c)
    grp, off = pos // span, pos % span
    gsz = np.minimum(G, bh - grp * G)
    present = off < gsz * nblk
    head = grp * G + off % np.maximum(gsz, 1)
    qb = nblk - 1 - off // np.maximum(gsz, 1)
    return cta[present], head[present], qb[present]


def _kv_bytes(n, d, qk, pv):
    return n * ((d / 2 + d / 16 if qk == "nvfp4" else d) + (d / 2 if pv == "nvfp4" else d))


CASES = [  # (B*H, N, d, qk, pv)
    (128, 4096, 128, "nvfp4", "fp8"),    # LLM prefill
    (1024, 2048, 128, "nvfp4", "fp8"),   # a partial last group
    (1024, 1024, 64, "fp8", "fp8"),
    (32, 131072, 128, "nvfp4", "fp8"),   # one head's K/V exceeds the share: no groups
    (35, 300, 128, "nvfp4", "fp8"),      # fewer items than SMs
    (256, 16384, 128, "fp8", "fp8"),
    (600, 4096, 64, "nvfp4", "nvfp4"),
    (1, 128, 128, "nvfp4", "fp8"),
]


@pytest.mark.parametrize("bh,n,d,qk,pv", CASES)
def test_every_item_dealt_once(bh, n, d, qk, pv):
    plan = fp.causal_plan(bh, n, d, qk, pv, sm_count=148)
    nblk = -(-n // 128)
    cta, head, qb = _walk(plan, bh, n)
    assert len(head) == bh * nblk
    ids = head.astype(np.int64) * nblk + qb
    assert np.array_equal(np.sort(ids), np.arange(bh * nblk))
    assert plan["ctas"] == min(148, bh * nblk)
    assert 0 <= cta.min() and cta.max() < plan["ctas"]


@pytest.mark.parametrize("bh,n,d,qk,pv", CASES)
def test_groups_fit_the_share_and_keep_the_balance(bh, n, d, qk, pv):
    plan = fp.causal_plan(bh, n, d, qk, pv, sm_count=148)
    nblk = -(-n // 128)
    G, C = plan["heads_per_group"], plan["ctas"]
    kv = _kv_bytes(n, d, qk, pv)
    if bh * kv <= L2_SHARE:
        assert G == bh  # everything fits already
    if G < bh:
        assert G * kv <= L2_SHARE
        assert plan["group_positions"] % (2 * C) == 0 and plan["positions"] % (2 * C) == 0
    else:
        assert plan["positions"] == bh * nblk
    # modelled per-CTA work (blocks of the row + one for the item) against the
    # ungrouped snake over the same items
    cta, head, qb = _walk(plan, bh, n)
    load = np.bincount(cta, weights=qb + 2.0, minlength=C)
    order = np.arange(bh * nblk)
    rnd, c = order // C, order % C
    cta0 = np.where(rnd % 2 == 1, C - 1 - c, c)
    load0 = np.bincount(cta0, weights=(nblk - 1 - order // bh) + 2.0, minlength=C)
    assert load.max() <= 1.005 * load0.max() + 1e-9
    assert load.sum() == pytest.approx(load0.sum())


def test_llm_prefill_groups():
    """B4 H32 N4096: 37 heads a group (each head's K/V 0.8 MB), four groups."""
    plan = fp.causal_plan(128, 4096, 128, "nvfp4", "fp8", sm_count=148)
    assert plan == {"heads_per_group": 37, "group_positions": 1184, "positions": 4144, "ctas": 148}


def test_plan_refusals():
    lib = fp.library()
    import ctypes
    out = [ctypes.c_int32(0) for _ in range(4)]
    refs = [ctypes.byref(v) for v in out]
    assert lib.fpattn_causal_plan(0, 128, 128, 2, 1, 148, *refs) == 1          # no heads
    assert lib.fpattn_causal_plan(8, 128, 96, 2, 1, 148, *refs) == 2           # d
    assert lib.fpattn_causal_plan(8, 128, 128, 0, 1, 148, *refs) == 1          # dtype
    assert lib.fpattn_causal_plan(70000, 128, 128, 2, 1, 148, *refs) == 2      # too many heads
    assert lib.fpattn_causal_plan(8, 128, 128, 2, 1, 148, None, *refs[1:]) == 1
