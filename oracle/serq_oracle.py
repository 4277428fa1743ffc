"""SERQ CPU oracle — TEST INFRASTRUCTURE ONLY.

A plain, slow, step-by-step CPU restatement of what the SERQ W4A4 linear
computes.  Only the tests, the package's ``smoke()`` self-check and the
benchmark's CPU-baseline leg may import it; the library path never does.
It shares no code with the CUDA path.

Sources (cited by page title and section):
  [notes]   "SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM
            Quantization" reading notes (dihengye.cn): 关键公式/基础量化,
            Stage 1 (SAF), Stage 2 (saliency-aware error reconstruction),
            量化推理 (quantized inference), Stage 3 (offline permutation).
  [gist-zh] technical summary (gist.science/zh): 2.1 静态激活展平,
            2.2 显著性感知误差重建, 2.3 离线权重置换, 3 主要贡献.
  [gist-pt] resumo técnico (gist.science/pt): 2. Metodologia items 1-3.
  [abstract] fugumt.com page with the arXiv abstract: W4A8 and W4A4 settings.
  [MX]      OCP Microscaling Formats (MX) Specification v1.0 — the pages only
            name MXFP4; its element (E2M1) and shared-scale (E8M0) rules come
            from this public specification.

Arithmetic conventions (the pages fix none of them; these are the readings
used everywhere in this repository):
  * every quantization decision is taken in IEEE float32 with one rounding
    per operation and no fused multiply-add: s = fp32(amax / 7),
    q = rne(fp32(x / s)) -- numpy float32 ops round exactly this way;
  * round-half-to-even for the INT4 grid and for E2M1 (ties go to the even
    code);
  * products are exact (small integers, or E2M1 values times powers of two),
    accumulated in int64-exact float64 (INT4) or float64 (MXFP4).

Parity pins: every function here is pinned by tests under tests/ against
closed forms, hand cases, invariants (r=0 is plain W4A4, R=0 when the salient
rows are on the grid, SAF/permutation identity, permutation invariance) and a
brute-force dequantize-then-loop matmul on tiny shapes.  The choice among the
readings of which Q(W_s) the residual subtracts, how the salient activation
slice is scaled, and how the SAF calibration set is drawn cannot be pinned by
any value the pages print (parity unpinned for those readings; the
computation under each reading is pinned).
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

F32 = np.float32
INT4_QMAX = 7                       # 2^(n-1) - 1 with n = 4  [notes, 基础量化]
INT8_QMAX = 127                     # n = 8: the activations of the W4A8 setting [abstract]
MX_BLOCK = 32                       # elements sharing one E8M0 scale  [MX]
E2M1_EMAX = 2                       # exponent of the largest E2M1 normal (6 = 1.5 * 2^2)  [MX]
E8M0_BIAS = 127                     # [MX]
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])  # magnitudes of codes 0..7  [MX]
INT_WEIGHT_FORMATS = ("int4", "w4a8")  # INT4 weights; activations INT4 or INT8


# ---------------------------------------------------------------------------
# rounding helpers
# ---------------------------------------------------------------------------

def bf16_rne(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bfloat16 (ties to even), returned as float32."""
    x = np.ascontiguousarray(x, dtype=F32)
    assert np.all(np.isfinite(x)), "non-finite input"
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(F32)


# ---------------------------------------------------------------------------
# A1: symmetric absmax n-bit integer quantizer  [notes, 基础量化]
#     X_q = clip(round(X / s)),  s = max|X| / (2^(n-1) - 1)
# n = 4 everywhere in W4A4; n = 8 for the activations of W4A8 [abstract].
# ---------------------------------------------------------------------------

def int_scale(absmax: np.ndarray, qmax: int) -> np.ndarray:
    """s = fp32(max|X| / qmax), qmax = 2^(n-1) - 1."""
    return (np.asarray(absmax, dtype=F32) / F32(qmax)).astype(F32)


def int_codes(x: np.ndarray, s: np.ndarray, qmax: int) -> np.ndarray:
    """q = clip(rne(fp32(x / s)), -qmax, qmax); all-zero codes where s == 0."""
    x = np.asarray(x, dtype=F32)
    s = np.asarray(s, dtype=F32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (x / s).astype(F32)
    q = np.rint(v)
    q = np.where(s > 0, q, 0.0)
    return np.clip(q, -qmax, qmax).astype(np.int8)


def quantize_int(x: np.ndarray, axis: int, qmax: int):
    """Per-slice symmetric n-bit along ``axis``: returns (codes int8, scale fp32)."""
    x = np.asarray(x, dtype=F32)
    s = int_scale(np.max(np.abs(x), axis=axis, keepdims=True), qmax)
    return int_codes(x, s, qmax), np.squeeze(s, axis=axis)


def int4_scale(absmax: np.ndarray) -> np.ndarray:
    """s = fp32(max|X| / 7)."""
    return int_scale(absmax, INT4_QMAX)


def int4_codes(x: np.ndarray, s: np.ndarray) -> np.ndarray:
    """q = clip(rne(fp32(x / s)), -7, 7); all-zero codes where s == 0."""
    return int_codes(x, s, INT4_QMAX)


def quantize_int4(x: np.ndarray, axis: int):
    """Per-slice symmetric INT4 along ``axis``: returns (codes int8, scale fp32)."""
    return quantize_int(x, axis, INT4_QMAX)


def quantize_int8(x: np.ndarray, axis: int):
    """Per-slice symmetric INT8 along ``axis`` (codes in [-127, 127])."""
    return quantize_int(x, axis, INT8_QMAX)


# ---------------------------------------------------------------------------
# A12: MXFP4 = E2M1 elements + one E8M0 scale per 32 elements  [MX]
# ---------------------------------------------------------------------------

def mx_scale_exponent(absmax: np.ndarray) -> np.ndarray:
    """Shared exponent E = floor(log2(absmax)) - emax(E2M1), clamped to [-127, 127].

    absmax == 0 gives E = -127 (the smallest scale; all codes are then 0).
    """
    a = np.asarray(absmax, dtype=np.float64)
    _, ex = np.frexp(a)                       # a = m * 2^ex, m in [0.5, 1)
    e = ex.astype(np.int64) - 1 - E2M1_EMAX   # floor(log2 a) = ex - 1
    e = np.where(a > 0, e, -E8M0_BIAS)
    return np.clip(e, -E8M0_BIAS, E8M0_BIAS).astype(np.int32)


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """Nearest E2M1 code for already-scaled values (ties to the even code).

    The magnitude is the grid point closest to |v| (values past 6 take 6, the
    largest finite E2M1 value); when |v| sits exactly half-way between two grid
    points the even code wins.  The sign bit is the IEEE sign bit of v.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    flat = a.reshape(-1)
    mag = np.empty(flat.shape, dtype=np.uint8)
    chunk = 1 << 20
    for lo in range(0, flat.size, chunk):
        d = np.abs(flat[lo:lo + chunk, None] - E2M1_GRID[None, :])
        dmin = d.min(axis=1, keepdims=True)
        is_min = d == dmin
        n_min = is_min.sum(axis=1)
        first = np.argmax(is_min, axis=1)            # lowest code at the minimum
        # a tie is always between two adjacent codes; keep the even one
        tie_pick = np.where(first % 2 == 0, first, first + 1)
        mag[lo:lo + chunk] = np.where(n_min == 2, tie_pick, first).astype(np.uint8)
    sign = np.signbit(v).reshape(-1).astype(np.uint8)
    return (mag | (sign << 3)).reshape(v.shape)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    val = E2M1_GRID[c & 7]
    return np.where(c & 8, -val, val)


def quantize_mxfp4_rows(x: np.ndarray, ncols: Optional[int] = None):
    """Quantize each row of x in consecutive 32-element blocks.

    Only the first ``ncols`` columns are quantized (default: all); a last block
    that is cut short is padded with zeros, which do not change its absmax.
    Returns (codes uint8 [rows, nblocks*32], E int32 [rows, nblocks]); padded
    positions hold code 0.
    """
    x = np.asarray(x, dtype=F32)
    rows, cols = x.shape
    n = cols if ncols is None else ncols
    nb = -(-n // MX_BLOCK)
    xp = np.zeros((rows, nb * MX_BLOCK), dtype=F32)
    xp[:, :n] = x[:, :n]
    blocks = xp.reshape(rows, nb, MX_BLOCK)
    E = mx_scale_exponent(np.max(np.abs(blocks), axis=2))
    # v = x * 2^-E is exact in float64 (and in float32)
    v = blocks.astype(np.float64) * np.ldexp(1.0, -E.astype(np.int64))[:, :, None]
    codes = e2m1_encode(v).reshape(rows, nb * MX_BLOCK)
    return codes, E


def mxfp4_dequant(codes: np.ndarray, E: np.ndarray) -> np.ndarray:
    """Exact float64 value of row-blocked MXFP4 data: e2m1(code) * 2^E."""
    rows, cols = codes.shape
    nb = cols // MX_BLOCK
    vals = e2m1_decode(codes).reshape(rows, nb, MX_BLOCK)
    return (vals * np.ldexp(1.0, E.astype(np.int64))[:, :, None]).reshape(rows, cols)


# ---------------------------------------------------------------------------
# A3: static activation flattening  [notes, Stage 1; gist-zh 2.1; gist-pt 2.1]
#     Y = X W = (X diag(s)^-1)(diag(s) W);  s_j = sqrt(max|X_j| / max|W_j|)
# ---------------------------------------------------------------------------

def calib_absmax(X: np.ndarray) -> np.ndarray:
    """a_j = max_t |X[t, j]| over the calibration tokens."""
    return np.max(np.abs(np.asarray(X, dtype=F32)), axis=0).astype(F32)


def saf_scales(act_absmax: np.ndarray, W: np.ndarray) -> np.ndarray:
    """s_j = sqrt(fp32(a_j / b_j)) with b_j = max_n |W[j, n]|; s_j = 1 if a_j or b_j is 0."""
    a = np.asarray(act_absmax, dtype=F32)
    b = np.max(np.abs(np.asarray(W, dtype=F32)), axis=1).astype(F32)
    ok = (a > 0) & (b > 0)
    with np.errstate(divide="ignore", invalid="ignore"):
        s = np.sqrt((a / b).astype(F32)).astype(F32)
    return np.where(ok, s, F32(1.0)).astype(F32)


# ---------------------------------------------------------------------------
# A4: saliency ordering  [notes, Stage 2: W^ = P diag(s) W = [W_s; W_r]]
# ---------------------------------------------------------------------------

def saliency_permutation(s: np.ndarray) -> np.ndarray:
    """perm[i] = original channel at permuted position i: s descending, ties by index."""
    return np.argsort(-np.asarray(s, dtype=F32), kind="stable").astype(np.int32)


def fold_weight(W: np.ndarray, s: np.ndarray, perm: np.ndarray, dtype=F32) -> np.ndarray:
    """W^[i, n] = s[perm[i]] * W[perm[i], n] (one rounding in ``dtype``)."""
    W = np.asarray(W, dtype=dtype)
    s = np.asarray(s, dtype=dtype)
    return (s[perm][:, None] * W[perm, :]).astype(dtype)


def fold_activation(X: np.ndarray, s: np.ndarray, perm: np.ndarray, round_bf16: bool = True,
                    dtype=F32) -> np.ndarray:
    """X^[m, i] = X[m, perm[i]] / s[perm[i]]: the producer's folded output.

    With the offline fold of [notes, Stage 3] the previous layer emits this
    directly; it is stored in bf16 (round to nearest even).
    """
    X = np.asarray(X, dtype=dtype)
    s = np.asarray(s, dtype=dtype)
    xh = (X[:, perm] / s[perm][None, :]).astype(dtype)
    return bf16_rne(xh) if round_bf16 else xh


# ---------------------------------------------------------------------------
# serq_prepare  [notes, Stage 1-3; gist-zh 2.2]
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Prepared:
    fmt: str
    K: int
    N: int
    r: int
    s: np.ndarray            # fp32 [K], original channel order
    perm: np.ndarray         # int32 [K]
    s_perm: np.ndarray       # fp32 [K], s[perm]
    inv_s: np.ndarray        # fp32 [K], 1 / s[perm]
    W_hat: np.ndarray        # fp32 [K, N]
    qw: np.ndarray           # INT4: int8 [N, K]; MXFP4: uint8 codes [N, K]
    sw: Optional[np.ndarray]  # INT4: fp32 [N]
    Ew: Optional[np.ndarray]  # MXFP4: int32 [N, K/32]
    R: np.ndarray            # fp32 [r, N]
    qR: np.ndarray           # INT4: int8 [N, r]; MXFP4: uint8 codes [N, nbR*32]
    sR: Optional[np.ndarray]  # INT4: fp32 [N]
    ER: Optional[np.ndarray]  # MXFP4: int32 [N, nbR]

    def deq_w(self) -> np.ndarray:
        """Dequantized main weight, [N, K] float64."""
        if self.fmt in INT_WEIGHT_FORMATS:
            return self.qw.astype(np.float64) * self.sw.astype(np.float64)[:, None]
        return mxfp4_dequant(self.qw, self.Ew)

    def deq_R(self) -> np.ndarray:
        """Dequantized residual, [N, r] float64."""
        if self.fmt in INT_WEIGHT_FORMATS:
            return self.qR.astype(np.float64) * self.sR.astype(np.float64)[:, None]
        return mxfp4_dequant(self.qR, self.ER)[:, : self.r]


def prepare(W: np.ndarray, r: int, fmt: str, act_absmax: Optional[np.ndarray] = None,
            s: Optional[np.ndarray] = None, columns: Optional[np.ndarray] = None) -> Prepared:
    """Offline SERQ preparation of one linear (W is K x N, Y = X W).

    1. SAF scales s from calibration absmax (or given s)       [notes, Stage 1]
    2. saliency permutation, s descending                       [notes, Stage 2]
    3. W^ = P diag(s) W                                        [notes, Stage 2]
    4. RTN quantization of W^: INT4 per output channel over K,
       MXFP4 per 32 along K                                     [gist-zh 3 (RTN)]
    5. R = W^_s - Q(W^_s) on the first r rows, with Q the main
       weight quantization                                      [notes, Stage 2]
    6. Q(R): 4-bit, INT4 per output channel, MXFP4 per 32 along r  [gist-zh 2.2]

    fmt "w4a8" prepares the weight exactly as "int4" (4-bit weights, R 4-bit);
    only its activations differ (8-bit, see quant_act)            [abstract]

    ``columns`` restricts steps 3-6 to a subset of output channels (the
    quantization of each output channel is independent of the others); s and
    perm always use all of W.
    """
    assert fmt in ("int4", "w4a8", "mxfp4")
    W = np.asarray(W, dtype=F32)
    K, N = W.shape
    assert 0 <= r <= K
    if s is None:
        s = saf_scales(act_absmax, W)
    s = np.asarray(s, dtype=F32)
    perm = saliency_permutation(s)
    s_perm = s[perm]
    inv_s = (F32(1.0) / s_perm).astype(F32)
    Wc = W if columns is None else W[:, columns]
    W_hat = fold_weight(Wc, s, perm)                       # [K, Nc] fp32
    Wt = np.ascontiguousarray(W_hat.T)                     # [Nc, K]
    if fmt in INT_WEIGHT_FORMATS:
        qw, sw = quantize_int4(Wt, axis=1)                 # per output channel over K
        deq_s = (qw[:, :r].astype(F32) * sw[:, None]).astype(F32)
        R = (Wt[:, :r] - deq_s).astype(F32)                # [Nc, r]
        if r > 0:
            qR, sR = quantize_int4(R, axis=1)
        else:
            qR, sR = np.zeros((Wt.shape[0], 0), np.int8), np.zeros(Wt.shape[0], F32)
        return Prepared(fmt, K, N, r, s, perm, s_perm, inv_s, W_hat, qw, sw, None,
                        np.ascontiguousarray(R.T), qR, sR, None)
    qw, Ew = quantize_mxfp4_rows(Wt)                       # blocks of 32 along K
    if r > 0:
        nb_r = -(-r // MX_BLOCK)
        deq = (e2m1_decode(qw[:, : nb_r * MX_BLOCK]).reshape(-1, nb_r, MX_BLOCK)
               * np.ldexp(1.0, Ew[:, :nb_r].astype(np.int64))[:, :, None]).reshape(Wt.shape[0], -1)
        deq = deq[:, :r].astype(F32)                        # exact in fp32
        R = (Wt[:, :r] - deq).astype(F32)
        qR, ER = quantize_mxfp4_rows(R)
    else:
        R = np.zeros((Wt.shape[0], 0), F32)
        qR, ER = np.zeros((Wt.shape[0], 0), np.uint8), np.zeros((Wt.shape[0], 0), np.int32)
    return Prepared(fmt, K, N, r, s, perm, s_perm, inv_s, W_hat, qw, None, Ew,
                    np.ascontiguousarray(R.T), qR, None, ER)


# ---------------------------------------------------------------------------
# serq_quant_act: per-token activation quantization + salient slice
#   [notes, 基础量化 and 量化推理: X^_q and X~_{s,q}]
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class QuantAct:
    fmt: str
    r: int
    qx: np.ndarray            # INT4: int8 [M, K]; MXFP4: uint8 codes [M, K]
    sx: Optional[np.ndarray]  # INT4: fp32 [M]
    Ex: Optional[np.ndarray]  # MXFP4: int32 [M, K/32]
    qxs: np.ndarray           # INT4: int8 [M, r]; MXFP4: uint8 codes [M, nbr*32]
    sxs: Optional[np.ndarray]  # INT4: fp32 [M]
    Exs: Optional[np.ndarray]  # MXFP4: int32 [M, nbr]

    def deq_x(self) -> np.ndarray:
        if self.fmt in INT_WEIGHT_FORMATS:
            return self.qx.astype(np.float64) * self.sx.astype(np.float64)[:, None]
        return mxfp4_dequant(self.qx, self.Ex)

    def deq_xs(self) -> np.ndarray:
        if self.fmt in INT_WEIGHT_FORMATS:
            return self.qxs.astype(np.float64) * self.sxs.astype(np.float64)[:, None]
        return mxfp4_dequant(self.qxs, self.Exs)[:, : self.r]


def quant_act(Xhat: np.ndarray, r: int, fmt: str) -> QuantAct:
    """Quantize X^ per token and, under its own scale, the salient slice X^[:, :r]."""
    X = np.asarray(Xhat, dtype=F32)
    M, K = X.shape
    if fmt in INT_WEIGHT_FORMATS:
        qmax = INT8_QMAX if fmt == "w4a8" else INT4_QMAX
        qx, sx = quantize_int(X, 1, qmax)
        if r > 0:
            qxs, sxs = quantize_int(X[:, :r], 1, qmax)
        else:
            qxs, sxs = np.zeros((M, 0), np.int8), np.zeros(M, F32)
        return QuantAct(fmt, r, qx, sx, None, qxs, sxs, None)
    qx, Ex = quantize_mxfp4_rows(X)
    if r > 0:
        qxs, Exs = quantize_mxfp4_rows(X, ncols=r)
    else:
        qxs, Exs = np.zeros((M, 0), np.uint8), np.zeros((M, 0), np.int32)
    return QuantAct(fmt, r, qx, None, Ex, qxs, None, Exs)


# ---------------------------------------------------------------------------
# serq_linear: Y ~= X^_q W^_q + X~_{s,q} Q(R)   [notes, 量化推理]
# ---------------------------------------------------------------------------

def _exact_int_matmul(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Integer matmul a[M,K] @ b[K,N] via float64 (exact: |partial sums| << 2^53)."""
    assert a.shape[1] * 127 * 7 < 2 ** 52
    c = np.asarray(a, dtype=np.float64) @ np.asarray(b, dtype=np.float64)
    ci = c.astype(np.int64)
    assert np.array_equal(ci, c)
    return ci


@dataclasses.dataclass
class LinearOut:
    Y: np.ndarray                      # float64 [M, N]
    acc1: Optional[np.ndarray] = None  # INT4: int64 [M, N], sum_i qx * qw
    acc2: Optional[np.ndarray] = None  # INT4: int64 [M, N], sum_{i<r} qxs * qR


def linear(prep: Prepared, qa: QuantAct) -> LinearOut:
    """Main 4-bit product plus the single residual product, no intermediate quantization."""
    assert prep.fmt == qa.fmt and prep.r == qa.r
    if prep.fmt in INT_WEIGHT_FORMATS:
        acc1 = _exact_int_matmul(qa.qx, prep.qw.T)
        acc2 = _exact_int_matmul(qa.qxs, prep.qR.T) if prep.r > 0 else np.zeros_like(acc1)
        assert np.abs(acc1).max(initial=0) < 2 ** 31 and np.abs(acc2).max(initial=0) < 2 ** 31
        Y = (acc1 * qa.sx.astype(np.float64)[:, None] * prep.sw.astype(np.float64)[None, :]
             + acc2 * qa.sxs.astype(np.float64)[:, None] * prep.sR.astype(np.float64)[None, :])
        return LinearOut(Y, acc1, acc2)
    Y = qa.deq_x() @ prep.deq_w().T
    if prep.r > 0:
        Y = Y + qa.deq_xs() @ prep.deq_R().T
    return LinearOut(Y)


def serq_forward(X: np.ndarray, W: np.ndarray, r: int, fmt: str,
                 X_calib: Optional[np.ndarray] = None):
    """Whole pipeline on raw X (M x K) and W (K x N): calibrate, prepare, fold, quantize, multiply."""
    a = calib_absmax(X if X_calib is None else X_calib)
    prep = prepare(W, r, fmt, act_absmax=a)
    Xh = fold_activation(X, prep.s, prep.perm)
    qa = quant_act(Xh, r, fmt)
    return prep, Xh, qa, linear(prep, qa)


# ---------------------------------------------------------------------------
# Two-factor baseline (L2QER)  [notes, "L2QER 的双矩阵路径"; gist-zh 1; gist-pt 1]
#     Y^ = X_q W_q + Q(X_q L_{1,q}) L_{2,q}
# The error correction uses two low-rank factors, so the intermediate
# T = X_q L_{1,q} has to be quantized on the fly before the second product.
# Here both factors live in the same folded frame as W^ (L1's rows follow the
# SAF scales and permutation of the activations it multiplies), T leaves its
# product in bf16 (a linear's output), and Q is the activation quantizer of
# the format (per token for INT4, per 32 for MXFP4). SERQ's point of
# comparison: one more GEMM, one more quantization, a serial dependency.
# ---------------------------------------------------------------------------

def prepare_given_residual(W: np.ndarray, R_given: np.ndarray, fmt: str, act_absmax: Optional[np.ndarray] = None,
                           s: Optional[np.ndarray] = None) -> Prepared:
    """W^_q exactly as prepare(W, 0, fmt), with the residual slot holding Q(R_given)
    (R_given: k x N, quantized as Q(R) is) instead of W~_s - Q(W~_s)."""
    base = prepare(W, 0, fmt, act_absmax=act_absmax, s=s)
    R = np.asarray(R_given, dtype=F32)
    k = R.shape[0]
    Rt = np.ascontiguousarray(R.T)                        # [N, k]
    if fmt in INT_WEIGHT_FORMATS:
        qR, sR = quantize_int4(Rt, axis=1)
        return dataclasses.replace(base, r=k, R=R, qR=qR, sR=sR)
    qR, ER = quantize_mxfp4_rows(Rt)
    return dataclasses.replace(base, r=k, R=R, qR=qR, ER=ER)


def l2qer_linear(main: Prepared, l1: Prepared, qa: QuantAct, T_bf16: Optional[np.ndarray] = None) -> LinearOut:
    """Y = X_q W_q + Q(T) L_{2,q}, T = X_q L_{1,q} stored in bf16.

    main: prepare_given_residual(W, L2, ...); l1: prepare(L1, 0, ..., s = main.s)
    (L1 folded with the main weight's scales and permutation); qa: quant_act(X^, 0).
    T_bf16 replaces the bf16 intermediate (to check the later steps exactly)."""
    assert l1.r == 0 and qa.r == 0 and np.array_equal(l1.perm, main.perm)
    k = main.r
    T = bf16_rne(linear(l1, qa).Y.astype(F32)) if T_bf16 is None else np.asarray(T_bf16, dtype=F32)
    assert T.shape[1] == k
    qT = quant_act(T, k, main.fmt)                         # on-the-fly quantization of T
    res = QuantAct(main.fmt, k, qa.qx, qa.sx, qa.Ex, qT.qxs, qT.sxs, qT.Exs)
    return linear(main, res)


# ---------------------------------------------------------------------------
# Producers with the offline fold merged in  [notes, Stage 3 "行/列排列离线合并到
# 权重中"; gist-zh 2.3]: the layer that emits this linear's input writes X^
# (permuted, divided by s) directly, so the activation quantization can run in
# the same pass. In a LLaMA block the producers are RMSNorm (before q/k/v and
# gate/up) and SwiGLU (before down); the pages do not spell these layers out,
# so they are written here in their standard form.
# ---------------------------------------------------------------------------

def _f32_of_exact_sum(v: np.ndarray) -> np.float32:
    """float32 nearest to the exact sum of the float64 values v (ties to even)."""
    import math
    v = [float(t) for t in np.asarray(v, dtype=np.float64).reshape(-1)]
    d = math.fsum(v)                       # the exact sum, correctly rounded to float64
    f = np.float32(d)                      # float64 -> float32, nearest even
    if float(f) != d:
        # d may sit exactly half-way between two float32 values while the exact
        # sum does not: decide from the sign of the exact remainder
        lo, hi = (f, np.nextafter(f, np.float32(np.inf))) if float(f) < d else \
                 (np.nextafter(f, np.float32(-np.inf)), f)
        mid = (float(lo) + float(hi)) / 2.0    # exact in float64
        if d == mid:
            rem = math.fsum(v + [-mid])
            if rem > 0:
                f = hi
            elif rem < 0:
                f = lo
    return np.float32(f)


def rmsnorm_rstd(H: np.ndarray, eps: float) -> np.ndarray:
    """rstd[m] = 1 / sqrt(fp32(sum_j H[m,j]^2) / K + eps), each step one fp32 rounding.

    The sum of squares is the exact sum rounded once to fp32 (bf16 inputs square
    exactly in float64)."""
    H = np.asarray(H, dtype=F32)
    M, K = H.shape
    sq = H.astype(np.float64) ** 2
    ss = np.array([_f32_of_exact_sum(sq[m]) for m in range(M)], dtype=F32)
    ms = (ss / F32(K)).astype(F32)
    v = (ms + F32(eps)).astype(F32)
    return (F32(1.0) / np.sqrt(v).astype(F32)).astype(F32)


def rmsnorm_folded(H: np.ndarray, gamma: np.ndarray, eps: float, perm: np.ndarray,
                   inv_s: np.ndarray) -> np.ndarray:
    """RMSNorm producer with the fold:  X^[m, i] = bf16(fp32(H[m, perm[i]] * rstd[m])
    * fp32(gamma[perm[i]] * inv_s[i])).

    RMSNorm(h) = h / sqrt(mean(h^2) + eps) * gamma; its output channel perm[i]
    goes to position i divided by s[perm[i]] (1/s folded into gamma)."""
    H = np.asarray(H, dtype=F32)
    rstd = rmsnorm_rstd(H, eps)
    g = (np.asarray(gamma, dtype=F32)[perm] * np.asarray(inv_s, dtype=F32)).astype(F32)
    t = (H[:, perm] * rstd[:, None]).astype(F32)
    return bf16_rne((t * g[None, :]).astype(F32))


def swiglu_folded(Ygu: np.ndarray, perm: np.ndarray, inv_s: np.ndarray) -> np.ndarray:
    """SwiGLU producer with the fold, in float64 (no storage rounding):
    X^[m, i] = silu(g) * u / s, with g = Ygu[m, perm[i]], u = Ygu[m, F + perm[i]],
    silu(g) = g / (1 + exp(-g)); Ygu = [gate | up] outputs, F columns each."""
    Y = np.asarray(Ygu, dtype=np.float64)
    F = Y.shape[1] // 2
    g = Y[:, :F][:, perm]
    u = Y[:, F:][:, perm]
    with np.errstate(over="ignore"):
        silu = g / (1.0 + np.exp(-g))
    return silu * u * np.asarray(inv_s, dtype=np.float64)[None, :]


# ---------------------------------------------------------------------------
# The block around the SERQ linears (context for the time-to-first-token the
# pages report for a LLaMA-3-8B 2K prefill  [notes, GPU 性能分析]): rotary
# position embedding and causal grouped-query attention, both in float64.
# The pages do not restate these layers; they are written in their standard
# LLaMA form (rotate-half RoPE, softmax(q k^T / sqrt(d)) v with a causal mask,
# query head h reading key/value head h // (n_q / n_kv)).
# ---------------------------------------------------------------------------

def rope(x: np.ndarray, n_heads: int, head_dim: int, base: float, pos0: int = 0) -> np.ndarray:
    """Rotate-half RoPE of a token-major [M, n_heads * head_dim] array (float64):
    for pair i < d/2 of each head, angle = (pos0 + m) * base^(-2i/d),
    (x_i, x_{i+d/2}) -> (x_i cos - x_{i+d/2} sin, x_{i+d/2} cos + x_i sin)."""
    x = np.asarray(x, dtype=np.float64)
    M = x.shape[0]
    h = x.reshape(M, n_heads, head_dim)
    half = head_dim // 2
    inv_freq = np.power(float(base), -np.arange(0, head_dim, 2, dtype=np.float64) / head_dim)
    ang = (pos0 + np.arange(M, dtype=np.float64))[:, None] * inv_freq[None, :]
    c, sn = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x1, x2 = h[..., :half], h[..., half:]
    out = np.concatenate([x1 * c - x2 * sn, x2 * c + x1 * sn], axis=-1)
    return out.reshape(M, n_heads * head_dim)


def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, n_q: int, n_kv: int,
                     head_dim: int) -> np.ndarray:
    """softmax(q k^T / sqrt(d) + causal mask) v per query head, float64.
    q: [M, n_q*d], k, v: [M, n_kv*d] (token-major); returns [M, n_q*d]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    M = q.shape[0]
    group = n_q // n_kv
    out = np.zeros((M, n_q * head_dim))
    mask = np.triu(np.ones((M, M), dtype=bool), 1)
    for h in range(n_q):
        g = h // group
        qh = q[:, h * head_dim:(h + 1) * head_dim]
        kh = k[:, g * head_dim:(g + 1) * head_dim]
        vh = v[:, g * head_dim:(g + 1) * head_dim]
        S = qh @ kh.T / np.sqrt(head_dim)
        S[mask] = -np.inf
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P = P / P.sum(axis=1, keepdims=True)
        out[:, h * head_dim:(h + 1) * head_dim] = P @ vh
    return out


# ---------------------------------------------------------------------------
# canonical packed byte layouts used for bit-exact comparisons
# ---------------------------------------------------------------------------

def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte along the last axis: element 2j low nibble, 2j+1 high."""
    c = (np.asarray(codes).astype(np.int16) & 0xF).astype(np.uint8)
    if c.shape[-1] % 2:
        c = np.concatenate([c, np.zeros(c.shape[:-1] + (1,), np.uint8)], axis=-1)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def e8m0(E: np.ndarray) -> np.ndarray:
    """Biased E8M0 byte of a shared exponent."""
    return (np.asarray(E, dtype=np.int32) + E8M0_BIAS).astype(np.uint8)
