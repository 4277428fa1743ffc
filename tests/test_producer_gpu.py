"""Producers with the fold and the activation quantization fused (SERQ
reading notes Stage 3; gist.science/zh 2.3): serq_rmsnorm_quant_act and
serq_swiglu_quant_act against the oracle.

RMSNorm: the X^ copy and every packed code and scale bit-exact with
oracle.quant_act(oracle.rmsnorm_folded(...)). SwiGLU (its fp32 expf is not
bit-reproducible on the CPU): X^ within bf16 rounding of the oracle's float64
SwiGLU, and the codes and scales bit-exact with the oracle's quantization of
the kernel's own X^. Then producer -> serq_linear against the oracle chain.
"""

import numpy as np
import pytest
import torch

import w4a4_post_quantization_serq_b200 as S
from oracle import serq_oracle as O
from synth import activations, norm_weight, weights

from parity_util import compare_act, compare_y, to_dev_bf16

pytestmark = pytest.mark.gpu


def _weight(K, N, r, fmt, seed):
    """A prepared consumer linear (device) and the oracle's preparation of it."""
    Xc = activations(seed, 256, K, max(1, K // 100), "lognormal", 50.0)
    W = weights(seed + 1, K, N)
    a = O.calib_absmax(Xc)
    prep = O.prepare(W, r, fmt, act_absmax=a)
    w = S.serq_prepare(to_dev_bf16(W), r, fmt, act_absmax=torch.from_numpy(a).cuda())
    return w, prep


def _res(qa):
    return {"xq": qa.xq.cpu().numpy(), "xs": qa.xs.cpu().numpy(),
            "xsq": None if qa.xsq is None else qa.xsq.cpu().numpy(),
            "xss": None if qa.xss is None else qa.xss.cpu().numpy()}


RMS_CASES = [("int4", 64, 256, 256, 16), ("mxfp4", 64, 256, 256, 16), ("w4a8", 64, 256, 256, 16),
             ("w4a8", 65, 20480, 128, 40), ("int4", 77, 384, 256, 40),
             ("mxfp4", 77, 384, 256, 40), ("mxfp4", 5, 1024, 512, 0), ("int4", 33, 20480, 128, 128),
             ("mxfp4", 129, 4096, 256, 128),
             ("mxfp4", 1300, 1024, 256, 40),     # many rows, each shorter than the 512 chunks a CTA covers
             ("mxfp4", 40, 32768, 128, 128)]     # too wide to stage two rows: one row per CTA


@pytest.mark.parametrize("fmt,M,K,N,r", RMS_CASES)
def test_rmsnorm_quant_act(fmt, M, K, N, r):
    w, prep = _weight(K, N, r, fmt, 300 + K)
    H = activations(40 + M, M, K, max(1, K // 100), "lognormal", 20.0)
    H[min(3, M - 1)] = 0.0                               # a zero row: rstd = 1/sqrt(eps), X^ = 0
    gamma = norm_weight(50 + K, K)
    eps = 1e-5
    xh = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    qa = S.serq_rmsnorm_quant_act(w, to_dev_bf16(H), to_dev_bf16(gamma), eps, xhat=xh)
    S.serq_device_status()
    Xh = O.rmsnorm_folded(H, gamma, np.float32(eps), prep.perm, prep.inv_s)
    assert np.array_equal(xh.float().cpu().numpy().view(np.uint32), Xh.view(np.uint32)), "X^"
    compare_act(_res(qa), O.quant_act(Xh, r, fmt), M, K, r)
    # without the debug copy the codes and scales are the same
    qa2 = S.serq_rmsnorm_quant_act(w, to_dev_bf16(H), to_dev_bf16(gamma), eps)
    compare_act(_res(qa2), O.quant_act(Xh, r, fmt), M, K, r)


SWI_CASES = [("int4", 64, 256, 256, 16), ("mxfp4", 64, 256, 256, 16), ("w4a8", 77, 384, 256, 40),
             ("mxfp4", 77, 384, 256, 40),
             ("int4", 77, 384, 256, 40), ("mxfp4", 3, 1024, 512, 0), ("int4", 9, 20480, 128, 128)]


def _swiglu_check(fmt, M, F, N, r, seed):
    w, prep = _weight(F, N, r, fmt, 600 + F)
    g = activations(seed, M, F, max(1, F // 100), "const", 4.0) * np.float32(2.0)
    u = activations(seed + 1, M, F, max(1, F // 100), "lognormal", 20.0)
    Ygu = np.concatenate([g, u], axis=1).astype(np.float32)
    xh = torch.empty(M, F, dtype=torch.bfloat16, device="cuda")
    qa = S.serq_swiglu_quant_act(w, to_dev_bf16(Ygu), xhat=xh)
    S.serq_device_status()
    ref = O.swiglu_folded(Ygu, prep.perm, prep.inv_s)
    got = xh.float().cpu().numpy()
    # bf16 rounding (2^-9) + a few fp32 steps and expf's error
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-35), "X^ off by more than bf16 rounding"
    compare_act(_res(qa), O.quant_act(got, r, fmt), M, F, r)
    return w, prep, Ygu, qa, got


@pytest.mark.parametrize("fmt,M,F,N,r", SWI_CASES)
def test_swiglu_quant_act(fmt, M, F, N, r):
    _swiglu_check(fmt, M, F, N, r, 70 + M)


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "w4a8"])
def test_producer_then_linear(fmt):
    # RMSNorm -> gate/up-shaped linear, SwiGLU -> down-shaped linear
    M, K, F, r = 130, 512, 768, 32
    w1, p1 = _weight(K, 2 * F, r, fmt, 900)
    H = activations(91, M, K, 5, "lognormal", 20.0)
    gamma = norm_weight(92, K)
    qa1 = S.serq_rmsnorm_quant_act(w1, to_dev_bf16(H), to_dev_bf16(gamma), 1e-5)
    Y1 = S.serq_linear(w1, qa1)
    ref1 = O.linear(p1, O.quant_act(O.rmsnorm_folded(H, gamma, np.float32(1e-5), p1.perm, p1.inv_s), r, fmt))
    compare_y(Y1.float().cpu().numpy(), ref1.Y)
    w2, p2 = _weight(F, 256, r, fmt, 950)
    xh = torch.empty(M, F, dtype=torch.bfloat16, device="cuda")
    qa2 = S.serq_swiglu_quant_act(w2, Y1, xhat=xh)
    Y2 = S.serq_linear(w2, qa2)
    S.serq_device_status()
    ref2 = O.linear(p2, O.quant_act(xh.float().cpu().numpy(), r, fmt))
    compare_y(Y2.float().cpu().numpy(), ref2.Y)


@pytest.mark.slow
def test_full_size_producers():
    # LLaMA-3-8B MLP at M = 2048 (MXFP4, r = 128): RMSNorm -> gate/up input (K = 4096),
    # SwiGLU -> down input (F = 14336)
    M = 2048
    w, prep = _weight(4096, 256, 128, "mxfp4", 1300)
    H = activations(1301, M, 4096, 41, "lognormal", 20.0)
    gamma = norm_weight(1302, 4096)
    xh = torch.empty(M, 4096, dtype=torch.bfloat16, device="cuda")
    qa = S.serq_rmsnorm_quant_act(w, to_dev_bf16(H), to_dev_bf16(gamma), 1e-5, xhat=xh)
    S.serq_device_status()
    Xh = O.rmsnorm_folded(H, gamma, np.float32(1e-5), prep.perm, prep.inv_s)
    assert np.array_equal(xh.float().cpu().numpy().view(np.uint32), Xh.view(np.uint32))
    compare_act(_res(qa), O.quant_act(Xh, 128, "mxfp4"), M, 4096, 128)
    _swiglu_check("mxfp4", M, 14336, 256, 128, 1310)
