"""The LLaMA block around the SERQ linears (NEXT-3 context for the pages'
2K-prefill time to first token, reading notes "GPU 性能分析"): the attention,
RoPE, residual add and fold-quantize kernels against the float64 oracle, then
a whole block (RMSNorm -> qkv -> RoPE -> attention -> o -> add -> RMSNorm ->
gate/up with the SwiGLU epilogue -> down -> add) against the oracle's block.
"""

import numpy as np
import pytest
import torch

import w4a4_post_quantization_serq_b200 as S
from oracle import serq_oracle as O
from synth import activations, norm_weight, weights

from parity_util import compare_act, compare_y, to_dev_bf16

pytestmark = pytest.mark.gpu
D = 128


def _bf16(a):
    return O.bf16_rne(np.asarray(a, dtype=np.float32))


@pytest.mark.parametrize("M,nq,nkv", [(1, 2, 1), (64, 4, 2), (100, 4, 4), (257, 8, 2), (640, 4, 1)])
def test_attention_against_oracle(M, nq, nkv):
    qkv = activations(800 + M, M, (nq + 2 * nkv) * D, 4, "const", 3.0)
    dev = to_dev_bf16(qkv)
    q, k, v = dev[:, :nq * D], dev[:, nq * D:(nq + nkv) * D], dev[:, (nq + nkv) * D:]
    o = S.serq_attention_prefill(q, k, v, nq, nkv)
    S.serq_device_status()
    ref = O.causal_attention(qkv[:, :nq * D], qkv[:, nq * D:(nq + nkv) * D], qkv[:, (nq + nkv) * D:], nq, nkv, D)
    got = o.float().cpu().numpy()
    # P enters the second product in bf16, O is stored in bf16
    vmax = np.abs(qkv[:, (nq + nkv) * D:]).max()
    assert np.all(np.abs(got - ref) <= 2.0 ** -7 * np.abs(ref) + 8e-3 * vmax), float(np.abs(got - ref).max())


@pytest.mark.parametrize("M,heads,base,pos0", [(5, 2, 10000.0, 0), (300, 4, 500000.0, 0), (64, 1, 500000.0, 1000)])
def test_rope_against_oracle(M, heads, base, pos0):
    x = activations(900 + M, M, heads * D + 64, 2, "const", 5.0)      # extra columns stay untouched
    dev = to_dev_bf16(x)
    S.serq_rope(dev[:, :heads * D], heads, D, base, pos0)
    S.serq_device_status()
    got = dev.float().cpu().numpy()
    ref = O.rope(x[:, :heads * D], heads, D, base, pos0)
    assert np.all(np.abs(got[:, :heads * D] - ref) <= 2.0 ** -8 * np.abs(ref) + 2e-3 * np.abs(x).max())
    assert np.array_equal(got[:, heads * D:], x[:, heads * D:])


def test_add_is_bf16_of_the_fp32_sum():
    a = activations(1, 33, 512, 3, "const", 20.0)
    b = activations(2, 33, 512, 3, "lognormal", 20.0)
    got = S.serq_add(to_dev_bf16(a), to_dev_bf16(b)).float().cpu().numpy()
    assert np.array_equal(got.view(np.uint32), _bf16(a.astype(np.float32) + b.astype(np.float32)).view(np.uint32))


@pytest.mark.parametrize("fmt,M", [("int4", 77), ("mxfp4", 77), ("w4a8", 77), ("mxfp4", 1300)])
def test_fold_quant_act_bit_exact(fmt, M):
    K, r = 512, 40
    X = activations(3, M, K, 5, "lognormal", 30.0)
    W = weights(4, K, 256)
    a = O.calib_absmax(activations(5, 256, K, 5, "lognormal", 30.0))
    prep = O.prepare(W, r, fmt, act_absmax=a)
    w = S.serq_prepare(to_dev_bf16(W), r, fmt, act_absmax=torch.from_numpy(a).cuda())
    xh = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    qa = S.serq_fold_quant_act(w, to_dev_bf16(X), xhat=xh)
    S.serq_device_status()
    Xh = O.fold_activation(X, prep.s, prep.perm)
    assert np.array_equal(xh.float().cpu().numpy().view(np.uint32), Xh.view(np.uint32))
    res = {"xq": qa.xq.cpu().numpy(), "xs": qa.xs.cpu().numpy(), "xsq": qa.xsq.cpu().numpy(),
           "xss": qa.xss.cpu().numpy()}
    compare_act(res, O.quant_act(Xh, r, fmt), M, K, r)


def test_block_against_oracle():
    M, Hd, nq, nkv, F, r, eps, base = 200, 512, 4, 2, 768, 32, 1e-5, 500000.0
    nqkv = (nq + 2 * nkv) * D
    h0 = activations(10, M, Hd, 5, "lognormal", 10.0)
    g1, g2 = norm_weight(11, Hd), norm_weight(12, Hd)
    Wqkv, Wo, Wgu, Wd = weights(13, Hd, nqkv), weights(14, nq * D, Hd), weights(15, Hd, 2 * F), weights(16, F, Hd)
    cal = lambda seed, K: O.calib_absmax(activations(seed, 256, K, max(1, K // 100), "lognormal", 10.0))
    a_qkv, a_o, a_gu, a_d = cal(20, Hd), cal(21, nq * D), cal(22, Hd), cal(23, F)
    t = lambda a: torch.from_numpy(a).cuda()
    # GPU block
    w_qkv = S.serq_prepare(to_dev_bf16(Wqkv), r, "mxfp4", act_absmax=t(a_qkv))
    w_o = S.serq_prepare(to_dev_bf16(Wo), r, "mxfp4", act_absmax=t(a_o))
    w_d = S.serq_prepare(to_dev_bf16(Wd), r, "mxfp4", act_absmax=t(a_d))
    w_gu = S.serq_prepare_swiglu(to_dev_bf16(Wgu), r, w_d, act_absmax=t(a_gu))
    H0 = to_dev_bf16(h0)
    qkv = S.serq_linear(w_qkv, S.serq_rmsnorm_quant_act(w_qkv, H0, to_dev_bf16(g1), eps))
    S.serq_rope(qkv[:, :nq * D], nq, D, base)
    S.serq_rope(qkv[:, nq * D:(nq + nkv) * D], nkv, D, base)
    att = S.serq_attention_prefill(qkv[:, :nq * D], qkv[:, nq * D:(nq + nkv) * D], qkv[:, (nq + nkv) * D:], nq, nkv)
    H1 = S.serq_add(H0, S.serq_linear(w_o, S.serq_fold_quant_act(w_o, att)))
    hq = S.serq_linear_swiglu_quant(w_gu, S.serq_rmsnorm_quant_act(w_gu, H1, to_dev_bf16(g2), eps))
    H2 = S.serq_add(H1, S.serq_linear(w_d, hq))
    S.serq_device_status()
    # oracle block, float64 between the quantized steps, bf16 where the GPU stores
    p_qkv = O.prepare(Wqkv, r, "mxfp4", act_absmax=a_qkv)
    p_o = O.prepare(Wo, r, "mxfp4", act_absmax=a_o)
    p_gu = O.prepare(Wgu, r, "mxfp4", act_absmax=a_gu)
    p_d = O.prepare(Wd, r, "mxfp4", act_absmax=a_d)
    e = np.float32(eps)
    y = _bf16(O.linear(p_qkv, O.quant_act(O.rmsnorm_folded(h0, g1, e, p_qkv.perm, p_qkv.inv_s), r, "mxfp4")).Y)
    qr = _bf16(O.rope(y[:, :nq * D], nq, D, base))
    kr = _bf16(O.rope(y[:, nq * D:(nq + nkv) * D], nkv, D, base))
    o_att = _bf16(O.causal_attention(qr, kr, y[:, (nq + nkv) * D:], nq, nkv, D))
    yo = _bf16(O.linear(p_o, O.quant_act(O.fold_activation(o_att, p_o.s, p_o.perm), r, "mxfp4")).Y)
    h1 = _bf16(h0.astype(np.float32) + yo)
    ygu = O.linear(p_gu, O.quant_act(O.rmsnorm_folded(h1, g2, e, p_gu.perm, p_gu.inv_s), r, "mxfp4")).Y
    xd = _bf16(O.swiglu_folded(ygu, p_d.perm, p_d.inv_s))
    yd = _bf16(O.linear(p_d, O.quant_act(xd, r, "mxfp4")).Y)
    h2 = _bf16(h1.astype(np.float32) + yd)
    # the intermediate roundings and quantization decisions of the two paths can
    # differ near their boundaries; the block output agrees within 2 % of the row norm
    compare_y(H2.float().cpu().numpy(), h2.astype(np.float64), tol=2e-2)
    compare_y(H1.float().cpu().numpy(), h1.astype(np.float64), tol=2e-2)
