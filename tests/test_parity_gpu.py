"""GPU parity: every stage of the CUDA path against the CPU oracle.

Bit-exact: calibration absmax, SAF scales, permutation, 1/s, folded
activations, packed codes and scales of W^_q, Q(R), X^_q, X~_{s,q}, and the
int32 accumulators of the INT4-weight formats (W4A4 INT4 and W4A8). Within 2e-3 (max abs error over the row, divided by
the row's L2 norm): the bf16 output Y.
"""

import numpy as np
import pytest

from oracle import serq_oracle as O
from synth import activations, weights, workload

from parity_util import compare_act, compare_weight, compare_y, run_gpu

pytestmark = pytest.mark.gpu


def _check(X, W, r, fmt, X_calib=None):
    res = run_gpu(X, W, r, fmt, X_calib=X_calib)
    M, K = X.shape
    a = O.calib_absmax(X if X_calib is None else X_calib)
    assert np.array_equal(res["a"].view(np.uint32), a.view(np.uint32)), "calibration absmax"
    prep = O.prepare(W, r, fmt, act_absmax=a)
    compare_weight(res["view"], prep)
    Xh = O.fold_activation(X, prep.s, prep.perm)
    assert np.array_equal(res["Xh"].view(np.uint32), Xh.view(np.uint32)), "folded activations"
    qa = O.quant_act(Xh, r, fmt)
    compare_act(res, qa, M, K, r)
    out = O.linear(prep, qa)
    if fmt in ("int4", "w4a8"):
        assert np.array_equal(res["acc"][0], out.acc1), "acc1"
        assert np.array_equal(res["acc"][1], out.acc2), "acc2"
    return compare_y(res["Y"], out.Y)


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "w4a8"])
def test_tiny_workload(fmt):
    wl = workload("tiny_int4")
    lin = wl.linears[0]
    _check(lin.X(wl.M), lin.W(), lin.r, fmt)


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "w4a8"])
@pytest.mark.parametrize("M,K,N,r", [
    (1, 256, 256, 16),        # a single token
    (77, 384, 384, 32),       # ragged M, K % 256 == 128 (half K-tile), N % 256 == 128 (half N-tile)
    (200, 512, 640, 0),       # r = 0: plain W4A4
    (130, 1024, 512, 128),    # two M tiles, the pages' rank
    (64, 512, 256, 256),      # r = 256
    (129, 768, 1280, 40),     # r not a multiple of 32 (short salient block)
    (33, 256, 256, 256),      # r = K
    (300, 512, 512, 64),      # MXFP4 CTA pair whose second CTA has no rows (M % 256 <= 128)
    (257, 384, 384, 32),      # CTA pair with a half K-tile and a half N-tile
    (1024, 1024, 1536, 128),  # several pair tiles per cluster
])
def test_shapes(fmt, M, K, N, r):
    X = activations(1000 + M, M, K, max(1, K // 100), "lognormal", 50.0)
    W = weights(2000 + K, K, N)
    _check(X, W, r, fmt)


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "w4a8"])
def test_degenerate_rows(fmt):
    # a zero row, an all-equal row, a row with one huge outlier, exact ties
    M, K, N, r = 8, 256, 256, 16
    X = activations(7, M, K, 3, "const", 30.0)
    X[1] = 0.0
    X[2] = 1.5
    X[3] = 0.0
    X[3, 100] = 1000.0
    X[4, :] = np.where(np.arange(K) % 2 == 0, 3.5, -3.5)
    W = weights(8, K, N)
    W[5] = 0.0  # a zero weight row -> s_j = 1
    _check(X, W, r, fmt, X_calib=X)


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "w4a8"])
def test_calibration_on_separate_draw(fmt):
    M, K, N, r = 16, 512, 256, 128
    X = activations(21, M, K, 5, "const", 50.0)
    Xc = activations(22, 300, K, 5, "const", 50.0)
    W = weights(23, K, N)
    _check(X, W, r, fmt, X_calib=Xc)


def test_residual_reduces_error_on_gpu():
    # same trend as the oracle: the salient correction lowers the layer error
    wl = workload("tiny_int4")
    lin = wl.linears[0]
    X, W = lin.X(wl.M), lin.W()
    ref = X.astype(np.float64) @ W.astype(np.float64)
    errs = [np.linalg.norm(run_gpu(X, W, r, "int4")["Y"] - ref) for r in (0, 16, 64)]
    assert errs[1] < errs[0] and errs[2] < errs[1]


@pytest.mark.parametrize("M,K,N,r", [
    (1, 4096, 1024, 128),     # the pages' rank, k/v shape at one token
    (4, 1024, 512, 128),      # 5 K-tiles over 5 splits
    (8, 512, 256, 64),
    (9, 768, 384, 0),         # r = 0, 16-token MMA with 7 padding tokens
    (16, 4096, 1024, 256),
    (16, 256, 128, 256),      # one K-tile each for main and residual
    (3, 1152, 256, 64),       # odd scale-atom counts: a main K-tile and the residual K-tile with one atom each
    (4, 32768, 256, 128),     # 129 K-tiles over 8 splits: ranges longer than a CTA's scale burst
    (16, 14336, 384, 128),    # down-projection depth, 3 output blocks
])
def test_decode_shapes(M, K, N, r):
    # small M takes the split-K streaming kernel (MXFP4)
    X = activations(3000 + M, M, K, max(1, K // 100), "const", 50.0)
    Xc = activations(3100 + M, 256, K, max(1, K // 100), "const", 50.0)
    W = weights(3200 + K, K, N)
    _check(X, W, r, "mxfp4", X_calib=Xc)


def test_decode_repeated_calls_identical():
    # the split-K tickets are reset by each call: repeated calls agree bit for bit
    import torch
    import w4a4_post_quantization_serq_b200 as S
    from parity_util import to_dev_bf16
    M, K, N, r = 16, 2048, 512, 128
    X = activations(41, M, K, 20, "const", 50.0)
    W = weights(42, K, N)
    w = S.serq_prepare(to_dev_bf16(W), r, "mxfp4", act_absmax=S.serq_calib_absmax(to_dev_bf16(X)))
    qa = S.serq_quant_act(S.serq_fold_producer(w, to_dev_bf16(X)), r, "mxfp4")
    ys = [S.serq_linear(w, qa).clone() for _ in range(3)]
    S.serq_device_status()
    assert all(torch.equal(ys[0], y) for y in ys[1:])
