"""The SwiGLU producer fused into the gate/up linear's epilogue (MXFP4,
CTA-pair kernel): the down linear's permutation folded into the gate/up
weight's output columns offline (reading notes Stage 3, "行/列排列离线合并到
权重中"; gist.science/zh 2.3), and the epilogue writing down's quantized input.

Checked against the oracle: the arranged gate/up weight bit for bit (its
preparation of the column-permuted weight); the epilogue's X^ within 2e-3 of
the row norm of the oracle's float64 SwiGLU of the float64 gate/up product;
the codes and scales bit-exact with the oracle's quantization of that X^; and
the down linear on them within 2e-3.
"""

import numpy as np
import pytest
import torch

import w4a4_post_quantization_serq_b200 as S
from oracle import serq_oracle as O
from synth import activations, weights
from w4a4_post_quantization_serq_b200 import _native as NAT

from parity_util import compare_act, compare_weight, compare_y, to_dev_bf16

pytestmark = pytest.mark.gpu


def _arranged_columns(perm_d, F):
    cols = []
    for t in range(F // 128):
        blk = perm_d[128 * t:128 * t + 128]
        cols.extend(blk.tolist())
        cols.extend((F + blk).tolist())
    return np.array(cols)


@pytest.mark.parametrize("M,K,F,N,r_gu,r_d", [
    (300, 512, 384, 256, 32, 40),      # ragged M (second CTA of the last pair partly empty), short slice block
    (257, 256, 256, 256, 0, 128),      # no gate/up residual
    (1024, 1024, 768, 512, 128, 128),  # several tiles per pair, the pages' rank
    (640, 512, 512, 256, 64, 256),     # slice over two tiles
])
def test_swiglu_epilogue_against_oracle(M, K, F, N, r_gu, r_d):
    X = activations(700 + M, M, K, max(1, K // 100), "lognormal", 40.0)
    W_gu = weights(701 + K, K, 2 * F)
    W_d = weights(702 + F, F, N)
    Hc = activations(703 + F, 256, F, max(1, F // 100), "lognormal", 20.0)
    a_d = O.calib_absmax(Hc)
    prep_d = O.prepare(W_d, r_d, "mxfp4", act_absmax=a_d)
    w_d = S.serq_prepare(to_dev_bf16(W_d), r_d, "mxfp4", act_absmax=torch.from_numpy(a_d).cuda())
    a_gu = O.calib_absmax(X)
    w_gu = S.serq_prepare_swiglu(to_dev_bf16(W_gu), r_gu, w_d, act_absmax=torch.from_numpy(a_gu).cuda())
    compare_weight({k: v.cpu().numpy() for k, v in w_gu.view().items()},
                   O.prepare(W_gu[:, _arranged_columns(prep_d.perm, F)], r_gu, "mxfp4", act_absmax=a_gu))

    qa = S.serq_quant_act(S.serq_fold_producer(w_gu, to_dev_bf16(X)), r_gu, "mxfp4")
    xh = torch.empty(M, F, dtype=torch.bfloat16, device="cuda")
    h = S.serq_linear_swiglu_quant(w_gu, qa, xhat=xh)
    Yd = S.serq_linear(w_d, h)
    S.serq_device_status()

    prep_gu = O.prepare(W_gu, r_gu, "mxfp4", act_absmax=a_gu)
    Ygu = O.linear(prep_gu, O.quant_act(O.fold_activation(X, prep_gu.s, prep_gu.perm), r_gu, "mxfp4")).Y
    got = xh.float().cpu().numpy()
    ref = O.swiglu_folded(Ygu, prep_d.perm, prep_d.inv_s)
    # X^ is stored in bf16: each element within twice bf16's half-ulp of the float64
    # value, plus a term for the fp32 accumulation of gate and up (relative to the row)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-4 * np.abs(ref).max(axis=1, keepdims=True)
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) / bound))
    qh = O.quant_act(got, r_d, "mxfp4")
    res = {"xq": h.xq.cpu().numpy(), "xs": h.xs.cpu().numpy(),
           "xsq": None if h.xsq is None else h.xsq.cpu().numpy(),
           "xss": None if h.xss is None else h.xss.cpu().numpy()}
    compare_act(res, qh, M, F, r_d)
    compare_y(Yd.float().cpu().numpy(), O.linear(prep_d, qh).Y)
    # without the debug copy the outputs are the same
    h2 = S.serq_linear_swiglu_quant(w_gu, qa)
    torch.cuda.synchronize()
    assert torch.equal(h2.xq, h.xq)


def test_swiglu_epilogue_small_m_is_refused():
    F = 256
    w_d = S.serq_prepare(to_dev_bf16(weights(1, F, 256)), 16, "mxfp4", s=torch.ones(F, device="cuda"))
    w_gu = S.serq_prepare_swiglu(to_dev_bf16(weights(2, 256, 2 * F)), 16, w_d, s=torch.ones(256, device="cuda"))
    qa = S.serq_quant_act(to_dev_bf16(activations(3, 128, 256, 2, "const", 10.0)), 16, "mxfp4")
    with pytest.raises(S.SerqError) as e:
        S.serq_linear_swiglu_quant(w_gu, qa)
    assert e.value.status == NAT.SERQ_EUNSUPPORTED
