"""The seeded input generators (synth/), which both the oracle and the CUDA
path read: shapes of the five workload configurations, determinism,
bf16 representability, the outlier-channel recipe and the bf16 rounding."""

import numpy as np
import pytest

from synth import activations, round_to_bf16, weights, workload
from synth.generators import bf16_bits


def _shapes(name, **kw):
    wl = workload(name, **kw)
    return wl.M, [(l.name, l.K, l.N, l.r, l.fmt) for l in wl.linears]


def test_config_shapes():
    assert _shapes("tiny_int4") == (64, [("tiny", 256, 256, 16, "int4")])
    assert _shapes("qproj_int4") == (2048, [("q_proj", 4096, 4096, 128, "int4")])
    # gate and up share one input: one prepared linear with N = 2 x 14336
    assert _shapes("mlp_mxfp4") == (2048, [("gate_up", 4096, 28672, 128, "mxfp4"),
                                           ("down", 14336, 4096, 128, "mxfp4")])
    M, lins = _shapes("decode_mxfp4")
    assert [(k, n) for _, k, n, _, _ in lins] == [(4096, 4096), (4096, 1024), (4096, 14336), (14336, 4096)]
    assert all(r == 128 and f == "mxfp4" for _, _, _, r, f in lins)
    for r in (0, 16, 128, 256):
        M, lins = _shapes("stack_mxfp4", r=r)
        assert M == 2048 and len(lins) == 32 * 4
        assert {(k, n) for _, k, n, _, _ in lins} == {(4096, 6144), (4096, 4096), (4096, 28672), (14336, 4096)}
        assert all(lr == r for _, _, _, lr, _ in lins)


def test_draws_are_deterministic_and_bf16():
    a1 = activations(7, 32, 256, 4, "const", 30.0)
    a2 = activations(7, 32, 256, 4, "const", 30.0)
    assert a1.dtype == np.float32 and np.array_equal(a1, a2)
    assert not np.array_equal(a1, activations(8, 32, 256, 4, "const", 30.0))
    w = weights(3, 256, 128)
    assert w.shape == (256, 128) and np.array_equal(w, weights(3, 256, 128))
    for t in (a1, w):
        bf16_bits(t)  # raises unless every value is bf16-representable
    # the weight draw does not depend on the activation draw of the same seed
    assert not np.allclose(weights(7, 32, 256).T[:32, :32], a1[:32, :32])


def test_outlier_channels():
    M, K, n = 512, 1024, 10
    x = activations(11, M, K, n, "const", 50.0)
    std = x.std(axis=0)
    big = np.flatnonzero(std > 10.0)
    assert len(big) == n                       # exactly n channels, drawn without replacement
    assert np.allclose(std[big], 50.0, rtol=0.1)
    assert np.all(std[std <= 10.0] < 1.3)
    xl = activations(11, M, K, n, "lognormal", 50.0)
    stdl = xl.std(axis=0)
    assert np.array_equal(np.flatnonzero(stdl > 5.0), big)  # same channels, lognormal magnitudes
    assert len(np.unique(np.round(stdl[big], 1))) > 1


def test_percent_outliers_of_the_configs():
    # 1 % of the input channels (round(0.01 K)): 41 of 4096, 143 of 14336
    for name, K, expect in (("qproj_int4", 4096, 41), ("decode_mxfp4", 14336, 143)):
        lin = [l for l in workload(name).linears if l.K == K][0]
        x = lin.X(256)
        assert int((x.std(axis=0) > 10.0).sum()) == expect


@pytest.mark.parametrize("x,expect", [
    (1.0 + 2.0 ** -8, 1.0),                      # tie -> even mantissa (down)
    (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),      # tie -> even mantissa (up)
    (1.0 + 2.0 ** -8 + 2.0 ** -20, 1.0 + 2.0 ** -7),  # above the tie
    (-(1.0 + 2.0 ** -8), -1.0),
    (65536.0 + 128.0, 65536.0),                  # spacing 512 at 2^16: nearest below
    (65536.0 + 256.0, 65536.0),                  # tie -> even (mantissa 0)
    (65536.0 + 768.0, 66560.0),                  # tie between mantissas 1 and 2 -> 2
    (0.0, 0.0),
])
def test_round_to_bf16_hand_cases(x, expect):
    got = round_to_bf16(np.array([x], dtype=np.float32))[0]
    assert got == np.float32(expect), (x, got)
