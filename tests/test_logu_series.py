"""The small-x series that the sampled-attention kernels use for log u (CPU).

For x = p^K below 1e-3 the kernels evaluate
  log u = log C(L,2) + 2 log x + (L-2) log1p(-x) + log1p(a3 r (1 + a4 r (1 + a5 r (1 + a6 r))))
with r = x / (1-x) and a_j = (L-j+1)/j, i.e. the binomial tail
sum_{j>=2} C(L,j) x^j (1-x)^(L-j) with its terms past j = 6 dropped.  The
claim stated beside the kernel code is that the dropped part is below 4e-7
relative for x < 1e-3 and L <= 255.  Checked here against the oracle's fp64
tail sum (its own code), in fp64 (truncation alone) and in fp32 (the
kernel's precision)."""
import math

import numpy as np
import pytest


def _series(x, L, dtype):
    x = dtype(x)
    one = dtype(1)
    a = [dtype((L - j + 1) / j) for j in (3, 4, 5, 6)]
    r = x / (one - x)
    tail = a[0] * r * (one + a[1] * r * (one + a[2] * r * (one + a[3] * r)))
    lnC2 = dtype(math.log(L * (L - 1) / 2))
    return float(lnC2 + dtype(2) * np.log(x) + dtype(L - 2) * np.log1p(-x) + np.log1p(tail))


@pytest.mark.parametrize("L", [75, 150, 255])
@pytest.mark.parametrize("x", [1e-6, 1e-4, 9.99e-4])
def test_truncated_series_matches_the_binomial_tail(oracle_mod, L, x):
    K = 8
    p = x ** (1.0 / K)
    exact = math.log(oracle_mod.sampling_prob(p, K, L))
    x_back = p ** K  # the oracle sees p; use the same x
    assert abs(_series(x_back, L, np.float64) - exact) < 4e-7
    # fp32 arithmetic adds rounding: still far inside the estimator's budget
    assert abs(_series(x_back, L, np.float32) - exact) < 5e-6


def test_dropping_the_sixth_term_would_break_the_bound(oracle_mod):
    """Without the j = 6 term the error at x = 1e-3, L = 255 is about 1e-5:
    the pin above would catch a series one term shorter."""
    L, K, x = 255, 8, 9.99e-4
    p = x ** (1.0 / K)
    xb = p ** K
    exact = math.log(oracle_mod.sampling_prob(p, K, L))
    a3, a4, a5 = (L - 2) / 3, (L - 3) / 4, (L - 4) / 5
    r = xb / (1 - xb)
    short = math.log(L * (L - 1) / 2) + 2 * math.log(xb) + (L - 2) * math.log1p(-xb) + \
        math.log1p(a3 * r * (1 + a4 * r * (1 + a5 * r)))
    assert abs(short - exact) > 4e-7

