"""The synthetic ablation runs end to end on a small case: every arm's loss
curve is finite and starts from the same point, and full-precision Adam
and 1-bit Adam both lower the loss."""
import math

import pytest

from error_compensated_bit_adam_b200 import ablation

pytestmark = pytest.mark.gpu


def test_ablation_small_case_runs():
    curves = ablation.run(n=4096 * 3, W=4, steps=60, warmup=12, noise=0.1, lr=1e-2, seed=3,
                          every=10)
    assert set(curves) == {"adam", "onebit", "ec_grad"}
    starts = {c[0] for c in curves.values()}
    assert len(starts) == 1
    for name, c in curves.items():
        assert len(c) == 7 and all(math.isfinite(x) for x in c), name
    assert curves["adam"][-1] < curves["adam"][0]
    assert curves["onebit"][-1] < curves["onebit"][0]
