"""Parity at the full workload sizes, in the launch configurations bench.py times.

Packed codes and scales (weights and activations) are compared in full and
bit for bit; Y and the INT4 accumulators on a seeded sample of token rows,
which the oracle computes row by row.
"""

import dataclasses

import numpy as np
import pytest
import torch

import w4a4_post_quantization_serq_b200 as S
from oracle import serq_oracle as O
from synth import workload

from parity_util import compare_act, compare_weight, compare_y, to_dev_bf16

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SAMPLE_ROWS = 48
_PREP = {}


def _oracle_prepare(lin, W, a_o):
    key = (lin.name, lin.K, lin.N, lin.r, lin.fmt, lin.w_seeds, lin.calib_seed, a_o.tobytes()[:64])
    if key not in _PREP:
        _PREP.clear()
        _PREP[key] = O.prepare(W, lin.r, lin.fmt, act_absmax=a_o)
    return _PREP[key]


def _full(lin, M, rows_sample):
    X, W, Xc = lin.X(M), lin.W(), lin.X_calib(M)
    Xd = to_dev_bf16(X)
    a = S.serq_calib_absmax(to_dev_bf16(Xc))
    w = S.serq_prepare(to_dev_bf16(W), lin.r, lin.fmt, act_absmax=a)
    Xh = S.serq_fold_producer(w, Xd)
    qa = S.serq_quant_act(Xh, lin.r, lin.fmt)
    acc = torch.zeros(2, M, lin.N, dtype=torch.int32, device="cuda") if lin.fmt in ("int4", "w4a8") else None
    Y = S.serq_linear(w, qa, acc_dbg=acc)
    S.serq_device_status()
    res = {k: (None if getattr(qa, k) is None else getattr(qa, k).cpu().numpy()) for k in ("xq", "xs", "xsq", "xss")}
    view = {k: v.cpu().numpy() for k, v in w.view().items()}
    # oracle
    a_o = O.calib_absmax(Xc)
    assert np.array_equal(a.cpu().numpy().view(np.uint32), a_o.view(np.uint32))
    prep = _oracle_prepare(lin, W, a_o)
    compare_weight(view, prep)
    Xh_o = O.fold_activation(X, prep.s, prep.perm)
    assert np.array_equal(Xh.float().cpu().numpy().view(np.uint32), Xh_o.view(np.uint32))
    qa_o = O.quant_act(Xh_o, lin.r, lin.fmt)
    compare_act(res, qa_o, M, lin.K, lin.r)
    rows = np.sort(np.random.default_rng(M + lin.K).choice(M, rows_sample, replace=False)) \
        if rows_sample < M else np.arange(M)
    sub = O.QuantAct(qa_o.fmt, qa_o.r, qa_o.qx[rows], None if qa_o.sx is None else qa_o.sx[rows],
                     None if qa_o.Ex is None else qa_o.Ex[rows], qa_o.qxs[rows],
                     None if qa_o.sxs is None else qa_o.sxs[rows], None if qa_o.Exs is None else qa_o.Exs[rows])
    out = O.linear(prep, sub)
    if lin.fmt in ("int4", "w4a8"):
        acc_np = acc.cpu().numpy()
        assert np.array_equal(acc_np[0][rows], out.acc1)
        assert np.array_equal(acc_np[1][rows], out.acc2)
    return compare_y(Y.float().cpu().numpy()[rows], out.Y)


def test_qproj_int4_full():
    wl = workload("qproj_int4")
    _full(wl.linears[0], wl.M, SAMPLE_ROWS)


def test_qproj_w4a8_full():
    # the W4A8 setting on the same LLaMA-2-7B q_proj shape (INT8 activations)
    wl = workload("qproj_int4")
    _full(dataclasses.replace(wl.linears[0], fmt="w4a8"), wl.M, SAMPLE_ROWS)


@pytest.mark.parametrize("name", ["gate_up", "down"])
def test_mlp_mxfp4_full(name):
    wl = workload("mlp_mxfp4")
    lin = [l for l in wl.linears if l.name == name][0]
    _full(lin, wl.M, SAMPLE_ROWS)


@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("name", ["q", "kv", "gate_up", "down"])
def test_decode_mxfp4_full(name, M):
    wl = workload("decode_mxfp4")
    lin = [l for l in wl.linears if l.name == name][0]
    _full(lin, M, M)


# The 32-block LLaMA-3-8B-shaped stack with its rank sweep r in {0, 16, 128,
# 256}: every swept r on the first block's qkv, the ends of the sweep on the
# other shapes (gate/up at r = 128 is the MLP case above), and two of the last
# block's linears (other seeds).
_STACK_CASES = ([(0, "qkv", r) for r in (0, 16, 128, 256)]
                + [(0, "o", 16), (0, "o", 256), (0, "gate_up", 256), (0, "down", 16), (0, "down", 256)]
                + [(31, "qkv", 128), (31, "o", 128)])


@pytest.mark.parametrize("blk,name,r", _STACK_CASES)
def test_stack_mxfp4_full(blk, name, r):
    wl = workload("stack_mxfp4", r=r)
    lin = [l for l in wl.linears if l.name == f"b{blk}.{name}"][0]
    assert lin.r == r
    _full(lin, wl.M, SAMPLE_ROWS)
