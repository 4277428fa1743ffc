"""The two-factor baseline (L2QER: Y = X_q W_q + Q(X_q L1_q) L2_q; reading
notes "L2QER 的双矩阵路径") on the GPU against the oracle.

Bit-exact: the main weight with L2 in its residual slot, L1 folded with the
main weight's scales and permutation, and the on-the-fly quantization of the
intermediate T (checked on the kernel's own bf16 T). Within 2e-3 of the row
norm: T itself and Y.
"""

import numpy as np
import pytest
import torch

import w4a4_post_quantization_serq_b200 as S
from oracle import serq_oracle as O
from synth import activations, weights

from parity_util import compare_act, compare_weight, compare_y, to_dev_bf16

pytestmark = pytest.mark.gpu


def _res(qa):
    return {"xq": qa.xq.cpu().numpy(), "xs": qa.xs.cpu().numpy(),
            "xsq": None if qa.xsq is None else qa.xsq.cpu().numpy(),
            "xss": None if qa.xss is None else qa.xss.cpu().numpy()}


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "w4a8"])
@pytest.mark.parametrize("M,K,N,k", [(200, 512, 384, 128), (5, 1024, 512, 128), (300, 768, 256, 256)])
def test_l2qer_against_oracle(fmt, M, K, N, k):
    X = activations(500 + M, M, K, max(1, K // 100), "lognormal", 40.0)
    W = weights(501 + K, K, N)
    L1 = weights(502 + K, K, k, 0.05)
    L2 = weights(503 + K, k, N, 0.01)
    a = O.calib_absmax(X)
    main_o = O.prepare_given_residual(W, L2, fmt, act_absmax=a)
    l1_o = O.prepare(L1, 0, fmt, s=main_o.s)

    main = S.serq_prepare(to_dev_bf16(W), k, fmt, act_absmax=torch.from_numpy(a).cuda(), R=to_dev_bf16(L2))
    l1 = S.serq_prepare(to_dev_bf16(L1), 0, fmt, s=main.view()["s"])
    compare_weight({kk: v.cpu().numpy() for kk, v in main.view().items()}, main_o)
    compare_weight({kk: v.cpu().numpy() for kk, v in l1.view().items()}, l1_o)

    qa = S.serq_quant_act(S.serq_fold_producer(main, to_dev_bf16(X)), 0, fmt)
    scratch = {"T": torch.empty(M, k, dtype=torch.bfloat16, device="cuda"), "tq": S.alloc_act(M, k, k, fmt)}
    Y = S.serq_linear_l2qer(main, l1, qa, scratch=scratch)
    S.serq_device_status()

    qa_o = O.quant_act(O.fold_activation(X, main_o.s, main_o.perm), 0, fmt)
    T = scratch["T"].float().cpu().numpy()
    compare_y(T, O.linear(l1_o, qa_o).Y)                         # T = X_q L1_q
    compare_act(_res(scratch["tq"]), O.quant_act(T, k, fmt), M, k, k)   # Q(T), bit-exact
    compare_y(Y.float().cpu().numpy(), O.l2qer_linear(main_o, l1_o, qa_o, T_bf16=T).Y)
