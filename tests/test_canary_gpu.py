"""Guard bytes around every caller-owned output buffer (the stand-in for a
memory checker, which is not available on these GPUs).

Each output buffer is carved out of a larger allocation whose GUARD bytes on
either side hold a fixed pattern. Every entry point that writes caller memory
runs at sizes with ragged edges: M beyond a tile, N = 384 (one and a half CTA-
pair tiles), r not a multiple of the 32-value block. Then the guards must
still hold the pattern, and the outputs must equal those of the same call
into plainly allocated buffers. The values themselves are checked against the
oracle by the parity tests. These tests check that nothing is written past an
output's documented size, including through a masked tail.
"""

import pytest
import torch

import w4a4_post_quantization_serq_b200 as S
from w4a4_post_quantization_serq_b200 import _native as NV
from synth import activations, norm_weight, weights

from parity_util import to_dev_bf16

pytestmark = pytest.mark.gpu

GUARD = 4096      # bytes on each side; keeps the buffer 16-byte (in fact 512-byte) aligned
FILL = 0xA5
D = 128


class Guarded:
    """`nbytes` of device memory between two GUARD-byte runs of FILL."""

    def __init__(self, nbytes: int, dtype=torch.uint8, shape=None):
        self.n = nbytes
        self.raw = torch.full((GUARD + (nbytes + 15) // 16 * 16 + GUARD,), FILL, dtype=torch.uint8, device="cuda")
        t = self.raw[GUARD:GUARD + nbytes].view(dtype)
        self.t = t.view(shape) if shape is not None else t

    def intact(self) -> bool:
        return bool((self.raw[:GUARD] == FILL).all()) and bool((self.raw[GUARD + self.n:] == FILL).all())


def _plain(nbytes: int, dtype=torch.uint8, shape=None) -> torch.Tensor:
    t = torch.full((nbytes,), FILL, dtype=torch.uint8, device="cuda").view(dtype)
    return t.view(shape) if shape is not None else t


def _acts(M, K, r, fmt):
    """(guarded QuantAct, its Guarded buffers, plain QuantAct), all bytes set to FILL."""
    sz = S.serq_act_buffer_sizes(M, K, r, fmt)
    names = ["xq", "xs", "xsq", "xss"]
    g = {n: Guarded(sz[n]) if sz[n] > 0 else None for n in names}
    p = {n: _plain(sz[n]) if sz[n] > 0 else None for n in names}
    f = NV.FMT[fmt]
    qa_g = S.QuantAct(M, K, r, f, *[None if g[n] is None else g[n].t for n in names])
    qa_p = S.QuantAct(M, K, r, f, *[p[n] for n in names])
    return qa_g, [b for b in g.values() if b is not None], qa_p


def _same_act(a, b):
    for n in ("xq", "xs", "xsq", "xss"):
        x, y = getattr(a, n), getattr(b, n)
        assert (x is None) == (y is None), n
        if x is not None:
            assert torch.equal(x, y), n


def _check(guards):
    S.serq_device_status()
    bad = [i for i, g in enumerate(guards) if not g.intact()]
    assert not bad, f"guard bytes overwritten around output buffer(s) {bad}"


def _bf16_out(M, N):
    return Guarded(M * N * 2, torch.bfloat16, (M, N)), _plain(M * N * 2, torch.bfloat16, (M, N))


def _weight(fmt, K, N, r, seed=7):
    Xc = to_dev_bf16(activations(seed, 256, K, max(1, K // 100), "lognormal", 30.0))
    return S.serq_prepare(to_dev_bf16(weights(seed + 1, K, N)), r, fmt, act_absmax=S.serq_calib_absmax(Xc))


@pytest.mark.parametrize("fmt", ["mxfp4", "int4", "w4a8"])
@pytest.mark.parametrize("M,K,r", [(1, 512, 40), (77, 1024, 16), (300, 4096, 128), (5, 512, 0)])
def test_quant_act_stays_in_bounds(fmt, M, K, r):
    X = to_dev_bf16(activations(30 + M, M, K, 4, "lognormal", 30.0))
    qa_g, guards, qa_p = _acts(M, K, r, fmt)
    S.serq_quant_act(X, r, fmt, out=qa_g)
    S.serq_quant_act(X, r, fmt, out=qa_p)
    _check(guards)
    _same_act(qa_g, qa_p)


LINEAR_CASES = [("mxfp4", M) for M in (1, 5, 16, 17, 70, 128, 129, 200, 300)] + \
               [(f, M) for f in ("int4", "w4a8") for M in (5, 200)]


@pytest.mark.parametrize("fmt,M", LINEAR_CASES)
def test_linear_stays_in_bounds(fmt, M):
    K, N, r = 1024, 384, 40
    w = _weight(fmt, K, N, r)
    qa = S.serq_quant_act(S.serq_fold_producer(w, to_dev_bf16(activations(40 + M, M, K, 6, "lognormal", 30.0))),
                          r, fmt)
    yg, yp = _bf16_out(M, N)
    S.serq_linear(w, qa, Y=yg.t)
    S.serq_linear(w, qa, Y=yp)
    _check([yg])
    assert torch.equal(yg.t, yp)


def test_noalloc_linear_stays_in_bounds():
    M, K, N, r = 5, 1024, 384, 40
    w = _weight("mxfp4", K, N, r)
    v = w.view()
    qa = S.serq_quant_act(S.serq_fold_producer(w, to_dev_bf16(activations(50, M, K, 6, "lognormal", 30.0))),
                          r, "mxfp4")
    yg, yp = _bf16_out(M, N)
    for Y in (yg.t, yp):
        S.serq_linear_small_m_noalloc(M, K, N, r, v["wq"], v["w_scale"], v.get("rq"), v.get("r_scale"), qa, Y)
    _check([yg])
    assert torch.equal(yg.t, yp)


@pytest.mark.parametrize("fmt", ["mxfp4", "int4"])
def test_producers_stay_in_bounds(fmt):
    M, K, F, r = 77, 1024, 768, 40
    w = _weight(fmt, K, 256, r)
    wd = _weight(fmt, F, 256, r, seed=9)
    H = to_dev_bf16(activations(60, M, K, 5, "lognormal", 10.0))
    gamma = to_dev_bf16(norm_weight(61, K))
    Ygu = to_dev_bf16(activations(62, M, 2 * F, 5, "lognormal", 3.0))
    guards = []

    # calibration absmax and the plain fold
    ag, ap = Guarded(K * 4, torch.float32), _plain(K * 4, torch.float32)
    S.serq_calib_absmax(H, out=ag.t)
    S.serq_calib_absmax(H, out=ap)
    fg, fp = _bf16_out(M, K)
    S.serq_fold_producer(w, H, dst=fg.t)
    S.serq_fold_producer(w, H, dst=fp)
    guards += [ag, fg]
    pairs = [(ag.t, ap), (fg.t, fp)]

    acts = []
    for call, kk in ((lambda o, x: S.serq_rmsnorm_quant_act(w, H, gamma, 1e-5, out=o, xhat=x), K),
                     (lambda o, x: S.serq_fold_quant_act(w, H, out=o, xhat=x), K),
                     (lambda o, x: S.serq_swiglu_quant_act(wd, Ygu, out=o, xhat=x), F)):
        qa_g, g, qa_p = _acts(M, kk, r, fmt)
        xg, xp = _bf16_out(M, kk)
        call(qa_g, xg.t)
        call(qa_p, xp)
        guards += g + [xg]
        pairs.append((xg.t, xp))
        acts.append((qa_g, qa_p))
    _check(guards)
    for a, b in pairs:
        assert torch.equal(a, b)
    for a, b in acts:
        _same_act(a, b)


@pytest.mark.parametrize("M", [129, 300])     # the CTA-pair kernel only (M > 128)
def test_swiglu_epilogue_stays_in_bounds(M):
    K, F, r = 1024, 768, 40
    wd = _weight("mxfp4", F, 256, r, seed=11)
    Xc = to_dev_bf16(activations(12, 256, K, 8, "lognormal", 30.0))
    wgu = S.serq_prepare_swiglu(to_dev_bf16(weights(13, K, 2 * F)), r, wd, act_absmax=S.serq_calib_absmax(Xc))
    qa = S.serq_quant_act(S.serq_fold_producer(wgu, to_dev_bf16(activations(14 + M, M, K, 8, "lognormal", 30.0))),
                          r, "mxfp4")
    qa_g, guards, qa_p = _acts(M, F, r, "mxfp4")
    xg, xp = _bf16_out(M, F)
    S.serq_linear_swiglu_quant(wgu, qa, out=qa_g, xhat=xg.t)
    S.serq_linear_swiglu_quant(wgu, qa, out=qa_p, xhat=xp)
    _check(guards + [xg])
    _same_act(qa_g, qa_p)
    assert torch.equal(xg.t, xp)


@pytest.mark.parametrize("fmt", ["mxfp4", "int4"])
def test_l2qer_stays_in_bounds(fmt):
    M, K, N, k = 200, 512, 384, 128
    X = activations(70, M, K, 5, "lognormal", 40.0)
    a = S.serq_calib_absmax(to_dev_bf16(X))
    main = S.serq_prepare(to_dev_bf16(weights(71, K, N)), k, fmt, act_absmax=a,
                          R=to_dev_bf16(weights(72, k, N, 0.01)))
    l1 = S.serq_prepare(to_dev_bf16(weights(73, K, k, 0.05)), 0, fmt, s=main.view()["s"])
    qa = S.serq_quant_act(S.serq_fold_producer(main, to_dev_bf16(X)), 0, fmt)
    tg, tp = _bf16_out(M, k)
    tq_g, guards, tq_p = _acts(M, k, k, fmt)
    yg, yp = _bf16_out(M, N)
    S.serq_linear_l2qer(main, l1, qa, Y=yg.t, scratch={"T": tg.t, "tq": tq_g})
    S.serq_linear_l2qer(main, l1, qa, Y=yp, scratch={"T": tp, "tq": tq_p})
    _check(guards + [tg, yg])
    assert torch.equal(tg.t, tp) and torch.equal(yg.t, yp)
    _same_act(tq_g, tq_p)


@pytest.mark.parametrize("M,nq,nkv", [(1, 2, 1), (200, 2, 1), (257, 4, 2)])
def test_block_kernels_stay_in_bounds(M, nq, nkv):
    qkv = to_dev_bf16(activations(80 + M, M, (nq + 2 * nkv) * D, 4, "const", 3.0))
    q, k, v = qkv[:, :nq * D], qkv[:, nq * D:(nq + nkv) * D], qkv[:, (nq + nkv) * D:]
    og, op = _bf16_out(M, nq * D)
    S.serq_attention_prefill(q, k, v, nq, nkv, out=og.t)
    S.serq_attention_prefill(q, k, v, nq, nkv, out=op)

    # RoPE in place on a guarded copy of q
    rg = Guarded(M * nq * D * 2, torch.bfloat16, (M, nq * D))
    rg.t.copy_(q)
    rp = q.clone()
    S.serq_rope(rg.t, nq, D, 500000.0)
    S.serq_rope(rp, nq, D, 500000.0)

    # residual add over n = M * nq * D values
    ag, ap = _bf16_out(M, nq * D)
    S.serq_add(q.contiguous(), rp, out=ag.t)
    S.serq_add(q.contiguous(), rp, out=ap)
    _check([og, rg, ag])
    assert torch.equal(og.t, op) and torch.equal(rg.t, rp) and torch.equal(ag.t, ap)
