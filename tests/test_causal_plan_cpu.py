"""Causal schedule of the attention kernel (host logic, no GPU).

fpattn_causal_plan reports how a causal launch deals its (head, query block)
items to the persistent CTAs: longest first, with the heads in groups whose
K/V fit a share of the L2 and each group padded to whole pairs of snake
rounds; or in pairs of query blocks (i and its mirror) head by head. These
tests walk the schedule by the rules the header states and check that every
item is dealt exactly once, that the schedule keeps the balance it promises,
and that a group's K/V bytes fit the share.
"""

import numpy as np
import pytest

import precision_attention_nvfp4_b200 as fp

L2_SHARE = 32 * 2**20


def _walk(plan, bh, n):
    """(cta, head, query block) of every position that holds an item."""
    nblk = -(-n // 128)
    C, total, P = plan["ctas"], plan["positions"], plan["pairs_per_head"]
    pos = np.arange(total)
    if P:
        # CTA c's round r is position 2*((r//2)*C + c) + r%2
        j, half = pos // 2, pos % 2
        cta = j % C
        head, i = j // P, j % P
        qb = np.where(half == 0, nblk - 1 - i, i)
        present = (half == 0) | (2 * i + 1 != nblk)
        return cta[present], head[present], qb[present]
    G, span = plan["heads_per_group"], plan["group_positions"]
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
    (1024, 1024, 64, "fp8", "fp8"),      # FP8: the snake, ungrouped
    (32, 131072, 128, "nvfp4", "fp8"),   # one head's K/V exceed the share: pairs
    (35, 300, 128, "nvfp4", "fp8"),      # fewer items than SMs
    (256, 16384, 128, "fp8", "fp8"),
    (600, 4096, 64, "nvfp4", "nvfp4"),
    (1, 128, 128, "nvfp4", "fp8"),
    (92, 6144, 128, "fp8", "fp8"),       # pairs, even block count
    (80, 12123, 128, "nvfp4", "fp8"),    # pairs, odd block count and a ragged tail
    (64, 8192, 128, "nvfp4", "fp8"),     # K/V under the whole L2: the snake, ungrouped
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
def test_schedule_fits_the_share_and_keeps_the_balance(bh, n, d, qk, pv):
    plan = fp.causal_plan(bh, n, d, qk, pv, sm_count=148)
    nblk = -(-n // 128)
    G, C, P = plan["heads_per_group"], plan["ctas"], plan["pairs_per_head"]
    kv = _kv_bytes(n, d, qk, pv)
    if bh * kv <= L2_SHARE:
        assert G == bh and P == 0  # everything fits already
    if bh * kv <= 4 * L2_SHARE or d != 128 or nblk < 32:
        assert P == 0              # pairs only at d = 128, 32+ blocks, K/V beyond the whole L2
    if qk != "nvfp4" or nblk > 32:
        assert G == bh             # head groups only for NVFP4 Q/K with at most 32 blocks
    if P:
        assert G == bh and P == (nblk + 1) // 2 and plan["positions"] == 2 * bh * P
    elif G < bh:
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
    assert load.max() <= (1.015 if P else 1.005) * load0.max() + 1e-9
    assert load.sum() == pytest.approx(load0.sum())


def test_pairs_keep_few_heads_in_flight():
    """In the paired order the items of one round come from a few
    consecutive heads: every pair of a round holds nblk + 1 key blocks."""
    plan = fp.causal_plan(256, 16384, 128, "fp8", "fp8", sm_count=148)
    P, C = plan["pairs_per_head"], plan["ctas"]
    assert P == 64
    j = np.arange(C)  # the pairs of the first scheduling round
    assert len(np.unique(j // P)) == 3
    assert np.all((128 - 1 - j % P) + 1 + (j % P) + 1 == 129)


def test_llm_prefill_groups():
    """B4 H32 N4096: 37 heads a group (each head's K/V 0.8 MB), four groups."""
    plan = fp.causal_plan(128, 4096, 128, "nvfp4", "fp8", sm_count=148)
    assert plan == {"heads_per_group": 37, "group_positions": 1184, "pairs_per_head": 0, "positions": 4144,
                    "ctas": 148}


def test_plan_refusals():
    lib = fp.library()
    import ctypes
    out = [ctypes.c_int32(0) for _ in range(5)]
    refs = [ctypes.byref(v) for v in out]
    assert lib.fpattn_causal_plan(0, 128, 128, 2, 1, 148, *refs) == 1          # no heads
    assert lib.fpattn_causal_plan(8, 128, 96, 2, 1, 148, *refs) == 2           # d
    assert lib.fpattn_causal_plan(8, 128, 128, 0, 1, 148, *refs) == 1          # dtype
    assert lib.fpattn_causal_plan(70000, 128, 128, 2, 1, 148, *refs) == 2      # too many heads
    assert lib.fpattn_causal_plan(8, 128, 128, 2, 1, 148, None, *refs[1:]) == 1
