"""Pins for the CPU oracle: hand cases, closed forms, invariants and brute force.

None of these re-types the oracle's own formulas; each checks the oracle
against a value or property fixed by the SERQ pages (or by the MX format the
pages name) so that a dropped term, a wrong sign, a wrong index or axis, or
a transposed operand in the oracle fails at least one test.
"""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import serq_oracle as O
from synth import activations, weights, workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# quantizer hand cases  (基础量化 formula; MX v1.0 E2M1/E8M0)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", _golden("quantizer_hand_cases.json")["int4"])
def test_int4_hand_cases(case):
    x = np.array([case["x"]], dtype=np.float32)
    q, s = O.quantize_int4(x, axis=1)
    assert float(s[0]) == case["scale"]
    assert q[0].tolist() == case["codes"]


@pytest.mark.parametrize("case", _golden("quantizer_hand_cases.json")["e2m1_block"])
def test_mxfp4_hand_cases(case):
    x = np.zeros((1, 32), dtype=np.float32)
    n = len(case["x"])
    x[0, :n] = case["x"]
    codes, E = O.quantize_mxfp4_rows(x)
    assert int(E[0, 0]) == case["E"]
    assert int(O.e8m0(E)[0, 0]) == case["e8m0"]
    assert codes[0, :n].tolist() == case["codes"]
    assert np.all(codes[0, n:] == 0)
    vals = O.mxfp4_dequant(codes, E)[0, :n]
    assert vals.tolist() == case["values"]
    assert np.array_equal(np.signbit(vals), np.signbit(np.array(case["values"])))


def test_e2m1_table_round_trip():
    # all 16 codes decode to the E2M1 values and encode back (except -0 -> -0)
    grid = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    for c in range(16):
        v = O.e2m1_decode(np.array([c], np.uint8))[0]
        mag = grid[c & 7]
        assert v == (-mag if c & 8 else mag)
        assert int(O.e2m1_encode(np.array([-0.0 if c == 8 else v]))[0]) == c


def test_e2m1_rounding_exhaustive_against_rational_nearest():
    # every float32 in a dense sweep of [-8, 8]: nearest grid point by exact
    # rational distance, ties to the even code
    grid = [Fraction(g) for g in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
    xs = np.concatenate([np.linspace(-8, 8, 4097, dtype=np.float32),
                         np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0, -0.25], np.float32),
                         np.nextafter(np.float32(0.25), np.float32(1))[None],
                         np.nextafter(np.float32(5.0), np.float32(0))[None]])
    codes = O.e2m1_encode(xs.astype(np.float64))
    for x, c in zip(xs.tolist(), codes.tolist()):
        a = abs(Fraction(x))
        d = [abs(a - g) for g in grid]
        best = min(d)
        cand = [i for i, di in enumerate(d) if di == best]
        mag = cand[0] if len(cand) == 1 else [i for i in cand if i % 2 == 0][0]
        assert c & 7 == mag, (x, c)
        assert (c >> 3) == (1 if math.copysign(1.0, x) < 0 else 0)


def test_mx_scale_exponent_closed_form():
    cases = {6.0: 0, 7.99: 0, 8.0: 1, 1.0: -2, 0.75: -3, 2.0 ** -120: -122,
             1e38: 124, 0.0: -127, 2.0 ** -126: -127, 2.0 ** -140: -127}
    for a, e in cases.items():
        assert int(O.mx_scale_exponent(np.array([a]))[0]) == e, a
    # after scaling, the block maximum lies in [4, 8): the E2M1 top binade
    rng = np.random.default_rng(7)
    a = np.abs(rng.standard_normal(1000)).astype(np.float32) * 10.0 ** rng.integers(-20, 20, 1000)
    a = a.astype(np.float32)
    a = a[a > 2.0 ** -120]
    E = O.mx_scale_exponent(a)
    v = a.astype(np.float64) * np.ldexp(1.0, -E.astype(np.int64))
    assert np.all((v >= 4) & (v < 8))


def test_int4_scale_axis_and_error_bound():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((9, 40)) * rng.uniform(0.1, 10, (9, 1))).astype(np.float32)
    q, s = O.quantize_int4(x, axis=1)
    for m in range(9):
        amax = max(abs(float(v)) for v in x[m])
        assert float(s[m]) == float(np.float32(amax) / np.float32(7))
        err = np.abs(x[m].astype(np.float64) - q[m].astype(np.float64) * float(s[m]))
        assert err.max() <= float(s[m]) / 2 * (1 + 1e-6)
    assert q.min() >= -7 and q.max() <= 7


def test_mxfp4_error_bound_and_grid():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((5, 128)) * 3).astype(np.float32)
    codes, E = O.quantize_mxfp4_rows(x)
    assert codes.max() <= 15 and np.all(O.e8m0(E) != 0xFF)
    d = O.mxfp4_dequant(codes, E)
    for m in range(5):
        for b in range(4):
            blk = x[m, 32 * b:32 * b + 32].astype(np.float64)
            unit = 2.0 ** int(E[m, b])
            # half the local grid step, or saturation at 6*2^E
            step = np.where(np.abs(blk) / unit < 2, 0.5, np.where(np.abs(blk) / unit < 4, 1.0, 2.0)) * unit
            err = np.abs(blk - d[m, 32 * b:32 * b + 32])
            sat = np.abs(blk) > 6 * unit
            assert np.all(err[~sat] <= step[~sat] / 2)
            assert np.all(np.abs(d[m, 32 * b:32 * b + 32][sat]) == 6 * unit)


def test_pack_nibbles_layout():
    codes = np.array([[1, 2, -1, 7, -7, 0]], np.int8)
    assert O.pack_nibbles(codes).tolist() == [[0x21, 0x7F, 0x09]]


# --------------------------------------------------------------------------
# SAF and permutation  (Stage 1 / Stage 2 / Stage 3)
# --------------------------------------------------------------------------

def test_saf_scale_closed_form_and_degenerate():
    a = np.array([4.0, 0.0, 9.0, 2.0], np.float32)
    W = np.array([[1.0, -1.0], [3.0, 0.5], [0.0, 0.0], [0.5, -0.125]], np.float32)
    s = O.saf_scales(a, W)
    assert s.tolist() == [2.0, 1.0, 1.0, 2.0]  # sqrt(4/1), a=0 -> 1, b=0 -> 1, sqrt(2/0.5)


def test_saliency_permutation_order_and_ties():
    s = np.array([1.0, 3.0, 2.0, 3.0, 0.5, 2.0], np.float32)
    perm = O.saliency_permutation(s)
    assert perm.tolist() == [1, 3, 2, 5, 0, 4]


def test_saf_and_permutation_identity_fp64():
    # (X diag(s)^-1 P^T)(P diag(s) W) = X W exactly up to fp64 rounding
    rng = np.random.default_rng(5)
    X = rng.standard_normal((7, 48))
    W = rng.standard_normal((48, 11))
    s = np.exp(rng.standard_normal(48))
    perm = O.saliency_permutation(s.astype(np.float32))
    Xh = O.fold_activation(X, s, perm, round_bf16=False, dtype=np.float64)
    Wh = O.fold_weight(W, s, perm, dtype=np.float64)
    ref = X @ W
    assert np.max(np.abs(Xh @ Wh - ref)) <= 1e-12 * np.max(np.abs(ref))
    # the salient block is the r rows with the largest s
    r = 5
    assert set(perm[:r].tolist()) == set(np.argsort(-s)[:r].tolist())


def test_permutation_invariance_int4_r0_bit_exact():
    # per-token / per-channel absmax are permutation-invariant and integer sums
    # commute, so the folded+permuted path equals the identity-permutation path
    X = activations(11, 16, 64, 2, "const", 30.0)
    W = weights(12, 64, 24)
    s = O.saf_scales(O.calib_absmax(X), W)
    prep = O.prepare(W, 0, "int4", s=s)
    qa = O.quant_act(O.fold_activation(X, prep.s, prep.perm), 0, "int4")
    out = O.linear(prep, qa)
    ident = np.arange(64, dtype=np.int32)
    Wh = O.fold_weight(W, s, ident)
    qw, sw = O.quantize_int4(np.ascontiguousarray(Wh.T), axis=1)
    Xh = O.bf16_rne((X / s[None, :]).astype(np.float32))
    qx, sx = O.quantize_int4(Xh, axis=1)
    acc = qx.astype(np.int64) @ qw.T.astype(np.int64)
    assert np.array_equal(out.acc1, acc)
    assert np.array_equal(qw[:, prep.perm], prep.qw) and np.array_equal(sw, prep.sw)


def test_permutation_invariance_mxfp4_up_to_quantization():
    X = activations(13, 8, 128, 2, "const", 50.0)
    W = weights(14, 128, 16)
    s = O.saf_scales(O.calib_absmax(X), W)
    prep = O.prepare(W, 0, "mxfp4", s=s)
    Y = O.linear(prep, O.quant_act(O.fold_activation(X, prep.s, prep.perm), 0, "mxfp4")).Y
    ident = O.fold_weight(W, s, np.arange(128))
    Xh = O.bf16_rne((X / s[None, :]).astype(np.float32))
    qx, Ex = O.quantize_mxfp4_rows(Xh)
    qw, Ew = O.quantize_mxfp4_rows(np.ascontiguousarray(ident.T))
    Y_id = O.mxfp4_dequant(qx, Ex) @ O.mxfp4_dequant(qw, Ew).T
    ref = X.astype(np.float64) @ W.astype(np.float64)
    # both are within the W4A4 quantization error of the exact product
    bound = 0.25 * np.linalg.norm(ref)
    assert np.linalg.norm(Y - ref) < bound and np.linalg.norm(Y_id - ref) < bound


# --------------------------------------------------------------------------
# the residual  R = W^_s - Q(W^_s)  and the runtime formula  (Stage 2, 量化推理)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", ["int4", "mxfp4"])
def test_residual_definition(fmt):
    W = weights(21, 96, 40)
    X = activations(22, 8, 96, 3, "const", 50.0)
    r = 32
    prep = O.prepare(W, r, fmt, act_absmax=O.calib_absmax(X))
    deq = prep.deq_w()                        # [N, K]
    # W^_s = Q(W^_s) + R on the r salient rows (exact up to one fp32 rounding)
    lhs = prep.W_hat[:r].astype(np.float64)
    rhs = deq[:, :r].T + prep.R.astype(np.float64)
    assert np.max(np.abs(lhs - rhs)) <= 2.0 ** -23 * np.max(np.abs(lhs))
    # rows beyond r carry no residual; R shrinks the salient-row error
    assert prep.R.shape == (r, 40)
    err_main = np.abs(lhs - deq[:, :r].T).sum()
    err_corr = np.abs(lhs - deq[:, :r].T - prep.deq_R().T).sum()
    assert err_corr < 0.5 * err_main


@pytest.mark.parametrize("fmt", ["int4", "mxfp4"])
def test_r0_is_plain_w4a4(fmt):
    # an independent plain W4A4 layer (per-token activations, per-channel or
    # per-32 weights), written with scalar loops
    X = activations(31, 4, 64, 2, "const", 30.0)
    W = weights(32, 64, 8)
    prep, Xh, qa, out = O.serq_forward(X, W, 0, fmt)
    M, K = Xh.shape
    N = W.shape[1]
    Wh = prep.W_hat
    Y = np.zeros((M, N))
    if fmt == "int4":
        sx = [np.float32(max(abs(float(v)) for v in Xh[m])) / np.float32(7) for m in range(M)]
        sw = [np.float32(max(abs(float(Wh[k, n])) for k in range(K))) / np.float32(7) for n in range(N)]
        for m in range(M):
            for n in range(N):
                acc = 0
                for k in range(K):
                    qx = max(-7, min(7, round(float(np.float32(Xh[m, k]) / sx[m]))))
                    qw = max(-7, min(7, round(float(np.float32(Wh[k, n]) / sw[n]))))
                    acc += qx * qw
                Y[m, n] = acc * float(sx[m]) * float(sw[n])
        assert np.array_equal(out.acc2, np.zeros_like(out.acc2))
    else:
        def mx(v):
            blocks = []
            for b in range(0, len(v), 32):
                blk = [float(t) for t in v[b:b + 32]]
                amax = max(abs(t) for t in blk)
                E = -127 if amax == 0 else max(-127, math.floor(math.log2(amax)) - 2)
                grid = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
                out_blk = []
                for t in blk:
                    a = abs(t) / 2.0 ** E
                    d = [abs(a - g) for g in grid]
                    c = [i for i, di in enumerate(d) if di == min(d)]
                    i = c[0] if len(c) == 1 else [j for j in c if j % 2 == 0][0]
                    out_blk.append(math.copysign(grid[i] * 2.0 ** E, t))
                blocks += out_blk
            return blocks
        dx = [mx(Xh[m]) for m in range(M)]
        dw = [mx(Wh[:, n]) for n in range(N)]
        for m in range(M):
            for n in range(N):
                Y[m, n] = sum(a * b for a, b in zip(dx[m], dw[n]))
    assert np.max(np.abs(out.Y - Y)) <= 1e-12 * np.max(np.abs(Y))


@pytest.mark.parametrize("fmt", ["int4", "mxfp4"])
def test_residual_vanishes_on_grid(fmt):
    # power-of-two SAF scales and salient rows of W^ exactly on the 4-bit grid
    # give R = 0, Q(R) = 0 and Y(r) == Y(0) bit for bit
    K, N, r, M = 128, 16, 32, 6
    rng = np.random.default_rng(41)
    s = (2.0 ** rng.integers(-2, 3, K)).astype(np.float32)
    s[:r] = 8.0                                  # the salient channels (largest s)
    s[r:] = np.minimum(s[r:], 4.0)
    Wh = np.zeros((K, N), np.float32)
    if fmt == "int4":
        # column amax 7 * 2^-3 -> s_w = 2^-3 exactly; salient rows are integer multiples
        Wh[:r] = rng.integers(-7, 8, (r, N)).astype(np.float32) * np.float32(0.125)
        Wh[0] = 7 * 0.125
        Wh[r:] = O.bf16_rne(rng.uniform(-0.8, 0.8, (K - r, N)).astype(np.float32))
    else:
        grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
        Wh[:r] = grid[rng.integers(0, 8, (r, N))] * np.where(rng.random((r, N)) < 0.5, -1, 1) * np.float32(2.0 ** -4)
        Wh[0] = 6 * 2.0 ** -4                    # block amax 6*2^-4 -> E = -4
        Wh[r:] = O.bf16_rne(rng.uniform(-0.3, 0.3, (K - r, N)).astype(np.float32))
    W = O.bf16_rne((Wh / s[:, None]).astype(np.float32))
    assert np.array_equal(W * s[:, None], Wh)    # exact: s are powers of two
    X = activations(42, M, K, 2, "const", 30.0)
    prep = O.prepare(W, r, fmt, s=s)
    assert np.array_equal(prep.perm[:r], np.arange(r))
    assert not np.any(prep.R) and not np.any(prep.deq_R())
    prep0 = O.prepare(W, 0, fmt, s=s)
    Xh = O.fold_activation(X, s, prep.perm)
    Y_r = O.linear(prep, O.quant_act(Xh, r, fmt)).Y
    Y_0 = O.linear(prep0, O.quant_act(Xh, 0, fmt)).Y
    assert np.array_equal(Y_r, Y_0)


@pytest.mark.parametrize("fmt,r,N", [("int4", 0, 7), ("int4", 16, 7), ("int4", 32, 7), ("mxfp4", 0, 7),
                                     ("mxfp4", 16, 7), ("mxfp4", 32, 7), ("mxfp4", 40, 7),
                                     ("int4", 16, 64), ("mxfp4", 16, 64)])
def test_brute_force_tiny(fmt, r, N):
    # dequantize every operand independently (table decode, per-element scale
    # lookup) and multiply with scalar loops; N == K catches a transposed weight
    M, K = 5, 64
    X = activations(51 + r, M, K, 2, "const", 30.0)
    W = weights(52 + r, K, N)
    prep, Xh, qa, out = O.serq_forward(X, W, r, fmt)
    grid = [0, 0.5, 1, 1.5, 2, 3, 4, 6]

    def dq_int4(code, scale):
        return float(int(code)) * float(scale)

    def dq_mx(code, E):
        c = int(code)
        v = grid[c & 7] * 2.0 ** int(E)
        return -v if c & 8 else v

    Y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                if fmt == "int4":
                    acc += dq_int4(qa.qx[m, k], qa.sx[m]) * dq_int4(prep.qw[n, k], prep.sw[n])
                else:
                    acc += dq_mx(qa.qx[m, k], qa.Ex[m, k // 32]) * dq_mx(prep.qw[n, k], prep.Ew[n, k // 32])
            for k in range(r):
                if fmt == "int4":
                    acc += dq_int4(qa.qxs[m, k], qa.sxs[m]) * dq_int4(prep.qR[n, k], prep.sR[n])
                else:
                    acc += dq_mx(qa.qxs[m, k], qa.Exs[m, k // 32]) * dq_mx(prep.qR[n, k], prep.ER[n, k // 32])
            Y[m, n] = acc
    assert np.max(np.abs(out.Y - Y)) <= 1e-12 * max(1e-300, np.max(np.abs(Y)))


def test_salient_slice_own_scale():
    X = activations(61, 6, 64, 2, "const", 30.0)
    Xh = O.bf16_rne(X)
    qa = O.quant_act(Xh, 16, "int4")
    for m in range(6):
        amax_s = max(abs(float(v)) for v in Xh[m, :16])
        assert float(qa.sxs[m]) == float(np.float32(amax_s) / np.float32(7))
    qm = O.quant_act(Xh, 16, "mxfp4")
    assert qm.qxs.shape == (6, 32) and np.all(qm.qxs[:, 16:] == 0)
    qm32 = O.quant_act(Xh, 32, "mxfp4")
    # r % 32 == 0: the salient blocks are the main blocks
    assert np.array_equal(qm32.qxs, qm32.qx[:, :32]) and np.array_equal(qm32.Exs, qm32.Ex[:, :1])


def test_zero_rows_give_zero():
    X = activations(71, 4, 64, 2, "const", 30.0)
    X[1] = 0
    for fmt in ("int4", "mxfp4"):
        prep, Xh, qa, out = O.serq_forward(X, weights(72, 64, 8), 16, fmt, X_calib=X)
        assert np.all(out.Y[1] == 0)


def test_error_reduction_with_rank():
    # the salient-row correction lowers the layer error (soft trend of the
    # rank ablation in '消融实验'); asserted on the tiny INT4 workload
    wl = workload("tiny_int4")
    lin = wl.linears[0]
    X, W = lin.X(wl.M), lin.W()
    ref = X.astype(np.float64) @ W.astype(np.float64)
    errs = []
    for r in (0, 16, 64):
        _, _, _, out = O.serq_forward(X, W, r, "int4")
        errs.append(np.linalg.norm(out.Y - ref))
    assert errs[1] < errs[0] and errs[2] < errs[1]


# --------------------------------------------------------------------------
# the pages' printed numbers (tests the page, not the kernel)
# --------------------------------------------------------------------------

def test_page_table_consistency():
    g = _golden("page_numbers.json")
    t = g["ttft_ms"]
    assert round(t["fp16"] / t["mxfp4"], 2) == g["speedup"]["mxfp4"]
    assert round(t["fp16"] / t["serq_mxfp4"], 2) == g["speedup"]["serq_mxfp4"]
    pm = g["peak_memory_gb"]
    assert round(pm["fp16"] / pm["serq_mxfp4"], 2) == pm["reduction"]
    # the table's own overhead (11.2%) is above the sentence's "<10%"
    assert t["serq_mxfp4"] / t["mxfp4"] - 1 > g["claimed_overhead_below"]
    assert 2 ** (g["bits"] - 1) - 1 == g["int4_divisor"] == O.INT4_QMAX
    ppl = g["rank_ppl"]
    assert ppl["0"] > ppl["16"] > ppl["128"] > ppl["256"]


# --------------------------------------------------------------------------
# hand values for the helpers every parity test relies on: the bf16 storage
# rounding of X^, the calibration maximum, the SAF divisor |W| and the
# salient slice's own scale (tests/golden/oracle_hand_cases.json)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", _golden("oracle_hand_cases.json")["bf16_rne"])
def test_bf16_rne_hand_cases(case):
    x = np.array([int(case["f32"], 16)], dtype=np.uint32).view(np.float32)
    got = O.bf16_rne(x).view(np.uint32)[0]
    assert got & 0xFFFF == 0
    assert int(got >> 16) == int(case["bf16"], 16), case["why"]


def test_calib_absmax_hand_values():
    g = _golden("oracle_hand_cases.json")["calib_absmax"]
    for xk, ak in (("X", "a"), ("X_square", "a_square")):
        a = O.calib_absmax(np.array(g[xk], np.float32))
        assert a.dtype == np.float32 and a.tolist() == g[ak]


def test_saf_scales_use_weight_magnitude():
    g = _golden("oracle_hand_cases.json")["saf_scales"]
    s = O.saf_scales(np.array(g["a"], np.float32), np.array(g["W"], np.float32))
    assert s.dtype == np.float32 and s.tolist() == g["s"], g["why"]


def _row(case):
    x = np.zeros((1, case["K"]), np.float32)
    for c, v in case["x_nonzero"].items():
        x[0, int(c)] = v
    return x


@pytest.mark.parametrize("case", _golden("oracle_hand_cases.json")["salient_slice"],
                         ids=lambda c: f"{c['fmt']}-r{c['r']}")
def test_salient_slice_hand_values(case):
    x = _row(case)
    qa = O.quant_act(x, case["r"], case["fmt"])
    if case["fmt"] == "mxfp4":
        assert qa.Ex[0].tolist() == case["E_main"]
        assert qa.Exs[0].tolist() == case["E_slice"], case["why"]
        assert qa.qxs.shape == (1, 32 * len(case["E_slice"]))
    else:
        assert float(qa.sx[0]) == case["scale_main"]
        assert float(qa.sxs[0]) == case["scale_slice"], case["why"]
        assert qa.qxs.shape == (1, case["r"])
    for c, code in case["codes_main_first"].items():
        assert int(qa.qx[0, int(c)]) == code, ("main", c)
    expect = np.zeros(qa.qxs.shape[1], np.int64)
    for c, code in case["codes_slice"].items():
        expect[int(c)] = code
    assert qa.qxs[0].astype(np.int64).tolist() == expect.tolist(), case["why"]


# --------------------------------------------------------------------------
# producers with the fold merged in (Stage 3): RMSNorm and SwiGLU
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", _golden("oracle_hand_cases.json")["exact_sum_to_f32"])
def test_exact_sum_rounds_once_to_f32(case):
    got = O._f32_of_exact_sum(np.array(case["v"], np.float64))
    assert got.dtype == np.float32 and float(got) == case["f32"], case["why"]


@pytest.mark.parametrize("case", _golden("oracle_hand_cases.json")["rmsnorm_folded"])
def test_rmsnorm_folded_hand_values(case):
    s = np.array(case["s"], np.float32)
    perm = O.saliency_permutation(s)
    inv_s = (np.float32(1) / s[perm]).astype(np.float32)
    H = np.array(case["H"], np.float32)
    assert O.rmsnorm_rstd(H, case["eps"]).tolist() == case["rstd"]
    got = O.rmsnorm_folded(H, np.array(case["gamma"], np.float32), case["eps"], perm, inv_s)
    assert got.tolist() == case["Xhat"], case["why"]


def test_rmsnorm_folded_against_textbook_rmsnorm():
    # h / sqrt(mean(h^2) + eps) * gamma in float64, then permuted and divided by s:
    # equal to the folded producer up to its fp32 steps and the final bf16 rounding
    rng = np.random.default_rng(9)
    M, K, eps = 6, 96, 1e-5
    H = O.bf16_rne((rng.standard_normal((M, K)) * rng.uniform(0.1, 30, (M, 1))).astype(np.float32))
    gamma = O.bf16_rne(rng.uniform(0.2, 2.0, K).astype(np.float32))
    s = np.exp(rng.standard_normal(K)).astype(np.float32)
    perm = O.saliency_permutation(s)
    inv_s = (np.float32(1) / s[perm]).astype(np.float32)
    Hd = H.astype(np.float64)
    ref = Hd / np.sqrt((Hd ** 2).mean(axis=1, keepdims=True) + eps) * gamma.astype(np.float64)
    ref = ref[:, perm] / s[perm].astype(np.float64)[None, :]
    got = O.rmsnorm_folded(H, gamma, eps, perm, inv_s).astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30)
    # scaling a row by a power of two leaves it unchanged (eps = 0)
    a = O.rmsnorm_folded(H, gamma, 0.0, perm, inv_s)
    b = O.rmsnorm_folded((H * np.float32(8)).astype(np.float32), gamma, 0.0, perm, inv_s)
    assert np.array_equal(a, b)
    # the fold: position i carries channel perm[i] (a one-hot row lands at perm^-1)
    one = np.zeros((1, K), np.float32)
    one[0, 17] = 1.0
    x = O.rmsnorm_folded(one, np.ones(K, np.float32), 0.0, perm, inv_s)
    pos = int(np.flatnonzero(x[0])[0])
    assert perm[pos] == 17 and np.count_nonzero(x) == 1


def test_swiglu_folded_closed_forms():
    g = np.array([0.0, math.log(3.0), -1000.0, 30.0])
    u = np.array([5.0, 2.0, 1.0, -1.0])
    Ygu = np.concatenate([g, u])[None, :]
    perm = np.arange(4)
    x = O.swiglu_folded(Ygu, perm, np.ones(4))[0]
    assert x[0] == 0.0                                         # silu(0) = 0
    assert abs(x[1] - 0.75 * math.log(3.0) * 2.0) < 1e-15     # exp(-ln 3) = 1/3: silu = g / (4/3)
    assert x[2] == 0.0                                         # exp overflow: g / inf = -0
    assert abs(x[3] + 30.0 / (1.0 + math.exp(-30.0))) < 1e-12
    # column mapping: gate channel perm[i] and up channel F + perm[i], divided by s
    Y = np.array([[1.0, 2.0, 3.0, 10.0, 20.0, 30.0]])
    perm = np.array([2, 0, 1])
    inv_s = np.array([0.5, 2.0, 4.0])
    got = O.swiglu_folded(Y, perm, inv_s)[0]
    silu = lambda t: t / (1.0 + math.exp(-t))
    want = [silu(3.0) * 30.0 * 0.5, silu(1.0) * 10.0 * 2.0, silu(2.0) * 20.0 * 4.0]
    assert np.allclose(got, want, rtol=1e-15, atol=0)


# --------------------------------------------------------------------------
# W4A8 (the abstract's second setting): INT4 weights and residual, INT8
# activations and salient slice, the same runtime formula
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", _golden("quantizer_hand_cases.json")["int8"])
def test_int8_hand_cases(case):
    q, s = O.quantize_int8(np.array([case["x"]], dtype=np.float32), axis=1)
    assert float(s[0]) == case["scale"]
    assert q[0].tolist() == case["codes"]


def test_w4a8_grid_and_weight_equal_to_int4():
    X = activations(81, 16, 128, 3, "lognormal", 50.0)
    W = weights(82, 128, 24)
    p8, Xh, qa, out = O.serq_forward(X, W, 32, "w4a8")
    p4 = O.prepare(W, 32, "int4", act_absmax=O.calib_absmax(X))
    # the weight side is the INT4 preparation, bit for bit
    for k in ("perm", "qw", "sw", "qR", "sR"):
        assert np.array_equal(getattr(p8, k), getattr(p4, k)), k
    assert qa.qx.min() >= -127 and qa.qx.max() <= 127 and qa.qx.dtype == np.int8
    assert np.abs(qa.qx).max() == 127                       # each row's absmax maps to 127
    sx = np.max(np.abs(Xh), axis=1) / np.float32(127)
    assert np.array_equal(qa.sx, sx.astype(np.float32))


def test_w4a8_r0_is_plain_w4a8_scalar_loops():
    X = activations(83, 4, 64, 2, "const", 30.0)
    W = weights(84, 64, 8)
    prep, Xh, qa, out = O.serq_forward(X, W, 0, "w4a8")
    M, K = Xh.shape
    N = W.shape[1]
    Wh = prep.W_hat
    for m in range(M):
        sx = np.float32(max(abs(float(v)) for v in Xh[m])) / np.float32(127)
        for n in range(N):
            sw = np.float32(max(abs(float(Wh[k, n])) for k in range(K))) / np.float32(7)
            acc = 0
            for k in range(K):
                qx = max(-127, min(127, round(float(np.float32(Xh[m, k]) / sx))))
                qw = max(-7, min(7, round(float(np.float32(Wh[k, n]) / sw))))
                acc += qx * qw
            assert out.acc1[m, n] == acc
            assert out.Y[m, n] == acc * float(sx) * float(sw)


def test_w4a8_brute_force_and_more_accurate_than_w4a4():
    wl = workload("tiny_int4")
    lin = wl.linears[0]
    X, W = lin.X(wl.M), lin.W()
    ref = X.astype(np.float64) @ W.astype(np.float64)
    errs = {}
    for fmt in ("int4", "w4a8"):
        prep, Xh, qa, out = O.serq_forward(X, W, 16, fmt)
        # dequantize every operand, multiply with a plain matmul: same Y
        Yb = qa.deq_x() @ prep.deq_w().T + qa.deq_xs() @ prep.deq_R().T
        assert np.max(np.abs(Yb - out.Y)) <= 1e-12 * np.max(np.abs(Yb))
        errs[fmt] = np.linalg.norm(out.Y - ref)
    assert errs["w4a8"] < errs["int4"]


# --------------------------------------------------------------------------
# the two-factor baseline (L2QER): Y = X_q W_q + Q(X_q L_{1,q}) L_{2,q}
# ("L2QER 的双矩阵路径"); SERQ's comparison point for the latency overhead
# --------------------------------------------------------------------------

def _l2qer_setup(fmt, K=128, N=48, k=32, seed=101):
    X = activations(seed, 12, K, 3, "lognormal", 40.0)
    W = weights(seed + 1, K, N)
    L1 = weights(seed + 2, K, k, 0.05)
    L2 = weights(seed + 3, k, N, 0.01)
    main = O.prepare_given_residual(W, L2, fmt, act_absmax=O.calib_absmax(X))
    l1 = O.prepare(L1, 0, fmt, s=main.s)
    qa = O.quant_act(O.fold_activation(X, main.s, main.perm), 0, fmt)
    return X, W, L1, L2, main, l1, qa


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "w4a8"])
def test_l2qer_zero_second_factor_is_plain_w4a4(fmt):
    X, W, L1, L2, main, l1, qa = _l2qer_setup(fmt)
    main0 = O.prepare_given_residual(W, np.zeros_like(L2), fmt, act_absmax=O.calib_absmax(X))
    plain = O.linear(O.prepare(W, 0, fmt, act_absmax=O.calib_absmax(X)), qa)
    assert np.array_equal(O.l2qer_linear(main0, l1, qa).Y, plain.Y)
    # the main weight is the r = 0 preparation bit for bit
    p0 = O.prepare(W, 0, fmt, act_absmax=O.calib_absmax(X))
    assert np.array_equal(main.qw, p0.qw) and np.array_equal(main.perm, p0.perm)


@pytest.mark.parametrize("fmt", ["int4", "mxfp4"])
def test_l2qer_brute_force(fmt):
    # every operand dequantized; T = X_q L1_q by a plain float64 matmul, rounded
    # to bf16, quantized per token (INT4) / per 32 (MXFP4); then both products
    X, W, L1, L2, main, l1, qa = _l2qer_setup(fmt)
    T = qa.deq_x() @ l1.deq_w().T                               # [M, k] in the folded frame
    T16 = O.bf16_rne(T.astype(np.float32))
    if fmt == "int4":
        q, s_ = O.quantize_int4(T16, axis=1)
        Tq = q.astype(np.float64) * s_.astype(np.float64)[:, None]
        L2q = O.quantize_int4(np.ascontiguousarray(L2.T), axis=1)
        L2d = L2q[0].astype(np.float64) * L2q[1].astype(np.float64)[:, None]
    else:
        c, E = O.quantize_mxfp4_rows(T16)
        Tq = O.mxfp4_dequant(c, E)
        c2, E2 = O.quantize_mxfp4_rows(np.ascontiguousarray(L2.T))
        L2d = O.mxfp4_dequant(c2, E2)
    Y = qa.deq_x() @ main.deq_w().T + Tq @ L2d.T
    got = O.l2qer_linear(main, l1, qa).Y
    assert np.max(np.abs(got - Y)) <= 1e-12 * np.max(np.abs(Y))
    # L1 is folded like W: the same product in the original frame
    Xd = X.astype(np.float64)
    assert np.allclose((Xd / main.s[None, :])[:, main.perm] @ l1.W_hat.astype(np.float64),
                       Xd @ L1.astype(np.float64), rtol=1e-5, atol=1e-6)


def test_l2qer_with_svd_factors_reduces_error():
    # factors from the truncated SVD of the folded weight's quantization error
    wl = workload("tiny_int4")
    lin = wl.linears[0]
    X, W = lin.X(wl.M), lin.W()
    a = O.calib_absmax(X)
    p0 = O.prepare(W, 0, "int4", act_absmax=a)
    E = p0.W_hat.astype(np.float64) - p0.deq_w().T                # [K, N], folded frame
    U, sv, Vt = np.linalg.svd(E, full_matrices=False)
    k = 16
    L1f = U[:, :k] * sv[:k]                                       # folded frame [K, k]
    L1 = np.zeros_like(L1f)
    L1[p0.perm] = L1f / p0.s[p0.perm].astype(np.float64)[:, None]  # back to the original frame
    L2 = Vt[:k]
    main = O.prepare_given_residual(W, L2.astype(np.float32), "int4", act_absmax=a)
    l1 = O.prepare(L1.astype(np.float32), 0, "int4", s=main.s)
    qa = O.quant_act(O.fold_activation(X, main.s, main.perm), 0, "int4")
    ref = X.astype(np.float64) @ W.astype(np.float64)
    err0 = np.linalg.norm(O.linear(p0, qa).Y - ref)
    err2 = np.linalg.norm(O.l2qer_linear(main, l1, qa).Y - ref)
    assert err2 < err0


# --------------------------------------------------------------------------
# the block around the linears (RoPE, causal GQA attention): closed forms
# --------------------------------------------------------------------------

def test_rope_closed_forms():
    rng = np.random.default_rng(41)
    nh, d = 3, 8
    x = rng.standard_normal((5, nh * d))
    y = O.rope(x, nh, d, 10000.0)
    assert np.array_equal(y[0], x[0])                        # position 0: no rotation
    # each (i, i + d/2) pair keeps its length
    xr, yr = x.reshape(5, nh, d), y.reshape(5, nh, d)
    n0 = xr[..., :4] ** 2 + xr[..., 4:] ** 2
    n1 = yr[..., :4] ** 2 + yr[..., 4:] ** 2
    assert np.allclose(n0, n1, rtol=1e-13)
    # pair 0 turns by exactly m radians (base^0 = 1): a complex multiplication
    m = 3
    z = (xr[m, :, 0] + 1j * xr[m, :, 4]) * np.exp(1j * m)
    assert np.allclose(yr[m, :, 0], z.real) and np.allclose(yr[m, :, 4], z.imag)
    # scores depend only on the relative position: shifting both by t changes nothing
    q, k = rng.standard_normal((1, d)), rng.standard_normal((1, d))
    def score(pq, pk, t):
        a = O.rope(q, 1, d, 500000.0, pos0=pq + t)
        b = O.rope(k, 1, d, 500000.0, pos0=pk + t)
        return float(a[0] @ b[0])
    assert abs(score(7, 2, 0) - score(7, 2, 100)) < 1e-9


def test_causal_attention_closed_forms():
    rng = np.random.default_rng(42)
    M, d, nq, nkv = 6, 4, 4, 2
    q = rng.standard_normal((M, nq * d))
    k = rng.standard_normal((M, nkv * d))
    v = rng.standard_normal((M, nkv * d))
    o = O.causal_attention(q, k, v, nq, nkv, d)
    # the first token sees only itself: its output is its own value row (of its kv head)
    for h in range(nq):
        g = h // 2
        assert np.allclose(o[0, h * d:(h + 1) * d], v[0, g * d:(g + 1) * d], rtol=1e-14)
    # zero queries: uniform weights over the visible prefix
    o0 = O.causal_attention(np.zeros_like(q), k, v, nq, nkv, d)
    for m in range(M):
        assert np.allclose(o0[m, :d], v[:m + 1, :d].mean(axis=0), rtol=1e-13)
    # query heads 0, 1 share kv head 0, heads 2, 3 share kv head 1
    q2 = q.copy()
    q2[:, d:2 * d] = q[:, :d]
    o2 = O.causal_attention(q2, k, v, nq, nkv, d)
    assert np.allclose(o2[:, :d], o2[:, d:2 * d])
    # a row is a convex combination of the visible values: inside their range
    vis_max = np.maximum.accumulate(v[:, :d], axis=0)
    assert np.all(o[:, :d] <= vis_max + 1e-12)
