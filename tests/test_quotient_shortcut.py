"""The INT4 / INT8 activation quantizers on the GPU take rint(fl(x / s)) (IEEE
division, ties to even, the oracle's decision) as rint(fl(x * fl(1 / s)))
whenever that product is more than 1e-4 away from a half-integer
(|q - rint(q)| < 0.4999), and divide only otherwise. For |x| <= max|x| = qmax * s the product is within 2^-22 of
x / s relative, so the two cannot round apart. Checked here in float32 on
random and exactly-tied quotients over the scale range.
"""

import numpy as np


def test_product_rounds_like_the_quotient_away_from_ties():
    rng = np.random.default_rng(7)
    checked = 0
    for qmax in (np.float32(7.0), np.float32(127.0)):
        for _ in range(12):
            amax = np.float32(10.0 ** rng.uniform(-30, 30))
            s = np.float32(amax / qmax)
            inv = np.float32(np.float32(1.0) / s)
            x = (rng.uniform(-1, 1, 50000).astype(np.float32) * amax).astype(np.float32)
            k = rng.integers(-2 * int(qmax), 2 * int(qmax) + 1, 5000).astype(np.float32)
            x = np.concatenate([x, (k * np.float32(0.5) * s).astype(np.float32)])  # exact ties
            x = x[np.abs(x) <= amax]
            q = (x * inv).astype(np.float32)
            fast = np.abs(q - np.rint(q)) < np.float32(0.4999)
            exact = np.rint((x / s).astype(np.float32))
            assert np.array_equal(np.rint(q[fast]), exact[fast])
            assert np.all(~fast[-5000:] | (np.rint(q[-5000:]) == exact[-5000:]))
            checked += int(fast.sum())
    assert checked > 1_000_000
