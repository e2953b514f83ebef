"""Denoising-step-aware schedule phases: TEST INFRASTRUCTURE ONLY.

FPSAttention page, section 3.2: over D denoising steps, thresholds
t1 = alpha1 * D and t2 = alpha2 * D split the process into three phases:
    t <= t1       early   (coarse quantization granularity, sparse window)
    t1 < t <= t2  middle  (fine granularity, dense window)
    t > t2        late    (intermediate granularity, medium window)
with alpha1 = 0.2 and alpha2 = 0.7 as the deployed values. Reading where the
page is silent: t counts the steps in the order they run, 1 .. D, and the
comparisons are made in float64.
"""
from __future__ import annotations

EARLY, MIDDLE, LATE = 0, 1, 2


def step_phase(t: int, D: int, alpha1: float = 0.2, alpha2: float = 0.7) -> int:
    assert 1 <= t <= D and 0.0 <= alpha1 <= alpha2 <= 1.0
    if t <= alpha1 * D:
        return EARLY
    if t <= alpha2 * D:
        return MIDDLE
    return LATE
