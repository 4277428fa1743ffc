"""The CTA-pair MXFP4 kernel on a grid of several rounds of 256 x 256 tiles
with a ragged last round (more tiles than co-resident pairs, not a multiple
of them) and a ragged M (the last pair's second CTA partly empty).

Y on seeded token rows against the oracle (row by row), every m-pair and
every output tile covered; a second call with other activations on the same
weight; two streams at once. The fused SwiGLU epilogue on the same tile
grid: its bf16 X^ on sampled rows against the oracle, and its quantized
outputs bit for bit against the quantization of its own X^ (all rows).
"""

import numpy as np
import pytest
import torch

import w4a4_post_quantization_serq_b200 as S
from oracle import serq_oracle as O
from synth import activations, weights

from parity_util import compare_act, compare_y, to_dev_bf16

pytestmark = pytest.mark.gpu

# 8 m-pairs (the last CTA partly empty) x 36 n-tiles = 288 tiles; 1024 + 128
# wide K = 5 K-tiles per tile
M, K, N, R = 1800, 1024, 9216, 128


def _rows(seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(M, 40, replace=False).tolist()) | {0, 255, 256, 1791, 1792, 1799}
    return np.array(sorted(rows))


def _oracle_rows(prep, Xh_o, rows, r, fmt):
    qa = O.quant_act(Xh_o[rows], r, fmt)
    return O.linear(prep, qa).Y


def _pairs():
    dev = torch.cuda.get_device_properties(0)
    return dev.multi_processor_count // 2


def test_grid_has_a_ragged_last_round():
    tiles = ((M + 255) // 256) * (N // 256)
    assert tiles > _pairs() and tiles % _pairs() != 0


def test_pair_grid_linear_against_oracle():
    W = weights(801, K, N)
    Xc = activations(802, 256, K, K // 100, "lognormal", 40.0)
    a = O.calib_absmax(Xc)
    prep = O.prepare(W, R, "mxfp4", act_absmax=a)
    w = S.serq_prepare(to_dev_bf16(W), R, "mxfp4", act_absmax=torch.from_numpy(a).cuda())
    for seed in (803, 804):
        X = activations(seed, M, K, K // 100, "lognormal", 40.0)
        qa = S.serq_quant_act(S.serq_fold_producer(w, to_dev_bf16(X)), R, "mxfp4")
        Y = S.serq_linear(w, qa)
        S.serq_device_status()
        rows = _rows(seed)
        ref = _oracle_rows(prep, O.fold_activation(X, prep.s, prep.perm), rows, R, "mxfp4")
        compare_y(Y.float().cpu().numpy()[rows], ref)


def test_pair_grid_two_streams():
    W = weights(811, K, N)
    a = O.calib_absmax(activations(812, 256, K, K // 100, "lognormal", 40.0))
    prep = O.prepare(W, R, "mxfp4", act_absmax=a)
    w = S.serq_prepare(to_dev_bf16(W), R, "mxfp4", act_absmax=torch.from_numpy(a).cuda())
    Xs = [activations(813 + i, M, K, K // 100, "lognormal", 40.0) for i in range(2)]
    qas = [S.serq_quant_act(S.serq_fold_producer(w, to_dev_bf16(X)), R, "mxfp4") for X in Xs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    Ys = [torch.empty(M, N, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    for _ in range(3):
        for i in range(2):
            with torch.cuda.stream(streams[i]):
                S.serq_linear(w, qas[i], Y=Ys[i])
    torch.cuda.synchronize()
    S.serq_device_status()
    for i in range(2):
        rows = _rows(820 + i)
        ref = _oracle_rows(prep, O.fold_activation(Xs[i], prep.s, prep.perm), rows, R, "mxfp4")
        compare_y(Ys[i].float().cpu().numpy()[rows], ref)


def test_pair_grid_swiglu_epilogue():
    F, N_d, r_d = N // 2, 512, 40
    X = activations(831, M, K, K // 100, "lognormal", 40.0)
    W_gu = weights(832, K, 2 * F)
    W_d = weights(833, F, N_d)
    a_d = O.calib_absmax(activations(834, 256, F, F // 100, "lognormal", 20.0))
    prep_d = O.prepare(W_d, r_d, "mxfp4", act_absmax=a_d)
    w_d = S.serq_prepare(to_dev_bf16(W_d), r_d, "mxfp4", act_absmax=torch.from_numpy(a_d).cuda())
    a_gu = O.calib_absmax(X)
    w_gu = S.serq_prepare_swiglu(to_dev_bf16(W_gu), R, w_d, act_absmax=torch.from_numpy(a_gu).cuda())
    qa = S.serq_quant_act(S.serq_fold_producer(w_gu, to_dev_bf16(X)), R, "mxfp4")
    xh = torch.empty(M, F, dtype=torch.bfloat16, device="cuda")
    h = S.serq_linear_swiglu_quant(w_gu, qa, xhat=xh)
    S.serq_device_status()
    got = xh.float().cpu().numpy()
    # X^ on sampled rows against the oracle's gate/up product and SwiGLU
    prep_gu = O.prepare(W_gu, R, "mxfp4", act_absmax=a_gu)
    rows = _rows(835)
    Ygu = _oracle_rows(prep_gu, O.fold_activation(X, prep_gu.s, prep_gu.perm), rows, R, "mxfp4")
    ref = O.swiglu_folded(Ygu, prep_d.perm, prep_d.inv_s)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-4 * np.abs(ref).max(axis=1, keepdims=True)
    assert np.all(np.abs(got[rows] - ref) <= bound), float(np.max(np.abs(got[rows] - ref) / bound))
    # every row's quantized output is the quantization of its own X^
    res = {"xq": h.xq.cpu().numpy(), "xs": h.xs.cpu().numpy(), "xsq": h.xsq.cpu().numpy(),
           "xss": h.xss.cpu().numpy()}
    compare_act(res, O.quant_act(got, r_d, "mxfp4"), M, F, r_d)
