"""Host learning-rate schedule (warmup + cosine), pinned by its closed forms
[CS336 §2 learning-rate schedule; LECTURE: max 6e-4, minimum 10% of it]."""
import math

import pytest

from decoder_only_lm_b200 import cosine_lr

MAX, MIN, W, TOT = 6e-4, 6e-5, 100, 1000


def test_warmup_is_linear_from_zero():
    assert cosine_lr(0, MAX, MIN, W, TOT) == 0.0
    assert cosine_lr(W // 2, MAX, MIN, W, TOT) == pytest.approx(MAX / 2, rel=1e-12)
    assert cosine_lr(1, MAX, MIN, W, TOT) == pytest.approx(MAX / W, rel=1e-12)


def test_cosine_end_points_and_midpoint():
    assert cosine_lr(W, MAX, MIN, W, TOT) == pytest.approx(MAX, rel=1e-12)
    mid = W + (TOT - W) // 2
    assert cosine_lr(mid, MAX, MIN, W, TOT) == pytest.approx((MAX + MIN) / 2, rel=1e-12)
    # a quarter of the way: cos(pi/4)
    q = W + (TOT - W) // 4
    want = MIN + (MAX - MIN) * (1 + math.cos(math.pi / 4)) / 2
    assert cosine_lr(q, MAX, MIN, W, TOT) == pytest.approx(want, rel=1e-12)


def test_floor_after_the_end_and_monotone_decay():
    assert cosine_lr(TOT, MAX, MIN, W, TOT) == MIN
    assert cosine_lr(10 * TOT, MAX, MIN, W, TOT) == MIN
    vals = [cosine_lr(t, MAX, MIN, W, TOT) for t in range(W, TOT + 1)]
    assert all(a >= b for a, b in zip(vals, vals[1:]))
    assert vals[-2] > MIN  # approaches the floor from above


def test_no_warmup_and_bad_arguments():
    assert cosine_lr(0, MAX, MIN, 0, TOT) == pytest.approx(MAX, rel=1e-12)
    for w, tot in ((-1, 10), (10, 10), (11, 10)):
        with pytest.raises(ValueError):
            cosine_lr(0, MAX, MIN, w, tot)
