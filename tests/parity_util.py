"""Helpers shared by the GPU parity tests: run the CUDA path, lay the oracle's
results out in the library's byte formats, compare."""

from __future__ import annotations

import numpy as np
import torch

from oracle import serq_oracle as O
import w4a4_post_quantization_serq_b200 as S

YTOL = 2e-3  # max_n |Y_gpu - Y_oracle| / ||Y_oracle[m, :]||_2, per row


def to_dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


def atoms_to_rows(buf: np.ndarray, rows: int, nblk: int) -> np.ndarray:
    """E8M0 bytes in the tensor-core atom layout -> [rows, nblk] array."""
    apr = (nblk + 3) // 4
    r = np.arange(rows)[:, None]
    b = np.arange(nblk)[None, :]
    off = ((r // 128) * apr + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)
    return buf[off]


def rp_of(r: int) -> int:
    return ((r + 63) // 64) * 64 if r > 0 else 0


def pad_cols(a: np.ndarray, width: int, fill=0) -> np.ndarray:
    out = np.full((a.shape[0], width), fill, dtype=a.dtype)
    out[:, : a.shape[1]] = a
    return out


def run_gpu(X: np.ndarray, W: np.ndarray, r: int, fmt: str, X_calib: np.ndarray = None, acc_dbg: bool = True):
    """Full CUDA path on device: calibrate, prepare, fold, quantize, linear."""
    Xd = to_dev_bf16(X)
    Wd = to_dev_bf16(W)
    Xc = Xd if X_calib is None else to_dev_bf16(X_calib)
    a = S.serq_calib_absmax(Xc)
    w = S.serq_prepare(Wd, r, fmt, act_absmax=a)
    Xh = S.serq_fold_producer(w, Xd)
    qa = S.serq_quant_act(Xh, r, fmt)
    M, N = X.shape[0], W.shape[1]
    acc = torch.zeros(2, M, N, dtype=torch.int32, device="cuda") if (acc_dbg and fmt in ("int4", "w4a8")) else None
    Y = S.serq_linear(w, qa, acc_dbg=acc)
    S.serq_device_status()
    view = w.view()
    res = {
        "a": a.cpu().numpy(), "Xh": Xh.float().cpu().numpy(), "Y": Y.float().cpu().numpy(),
        "view": {k: v.cpu().numpy() for k, v in view.items()},
        "xq": qa.xq.cpu().numpy(), "xs": qa.xs.cpu().numpy(),
        "xsq": None if qa.xsq is None else qa.xsq.cpu().numpy(),
        "xss": None if qa.xss is None else qa.xss.cpu().numpy(),
        "acc": None if acc is None else acc.cpu().numpy(),
        "weight": w, "qa": qa, "Xh_dev": Xh,
    }
    return res


def expected_weight_bytes(prep: O.Prepared):
    """The oracle's prepared weight in the library's byte layout."""
    r, rp = prep.r, rp_of(prep.r)
    N, K = prep.qw.shape
    out = {"perm": prep.perm, "s": prep.s, "inv_s": prep.inv_s, "wq": O.pack_nibbles(prep.qw)}
    if prep.fmt in O.INT_WEIGHT_FORMATS:
        out["w_scale"] = prep.sw
        if r > 0:
            out["rq"] = O.pack_nibbles(pad_cols(prep.qR, rp))
            out["r_scale"] = prep.sR
    else:
        out["w_scale_rows"] = O.e8m0(prep.Ew)
        if r > 0:
            out["rq"] = O.pack_nibbles(pad_cols(prep.qR, rp))
            out["r_scale_rows"] = O.e8m0(pad_cols(prep.ER, rp // 32, fill=-127))
    return out


def compare_weight(got: dict, prep: O.Prepared):
    exp = expected_weight_bytes(prep)
    v = got
    N, K = prep.qw.shape
    rp = rp_of(prep.r)
    assert np.array_equal(v["perm"], exp["perm"]), "perm"
    assert np.array_equal(v["s"].view(np.uint32), exp["s"].view(np.uint32)), "s"
    assert np.array_equal(v["inv_s"].view(np.uint32), exp["inv_s"].view(np.uint32)), "inv_s"
    assert np.array_equal(v["wq"], exp["wq"]), f"wq mismatch at {np.argwhere(v['wq'] != exp['wq'])[:5]}"
    if prep.fmt in O.INT_WEIGHT_FORMATS:
        assert np.array_equal(v["w_scale"].view(np.uint32), exp["w_scale"].view(np.uint32)), "sw"
        if prep.r > 0:
            assert np.array_equal(v["rq"], exp["rq"]), f"rq mismatch at {np.argwhere(v['rq'] != exp['rq'])[:5]}"
            assert np.array_equal(v["r_scale"].view(np.uint32), exp["r_scale"].view(np.uint32)), "sR"
    else:
        assert np.array_equal(atoms_to_rows(v["w_scale"], N, K // 32), exp["w_scale_rows"]), "w E8M0"
        if prep.r > 0:
            assert np.array_equal(v["rq"], exp["rq"]), f"rq mismatch at {np.argwhere(v['rq'] != exp['rq'])[:5]}"
            assert np.array_equal(atoms_to_rows(v["r_scale"], N, rp // 32), exp["r_scale_rows"]), "R E8M0"


def compare_act(res: dict, qa: O.QuantAct, M: int, K: int, r: int):
    rp = rp_of(r)
    if qa.fmt == "w4a8":  # one int8 code per element, fp32 scales
        xq = res["xq"][: M * K].reshape(M, K).view(np.int8)
        assert np.array_equal(xq, qa.qx), f"xq mismatch at {np.argwhere(xq != qa.qx)[:5]}"
        assert np.array_equal(res["xs"].view(np.float32)[:M].view(np.uint32), qa.sx.view(np.uint32)), "sx"
        if r > 0:
            xsq = res["xsq"][: M * rp].reshape(M, rp).view(np.int8)
            assert np.array_equal(xsq, pad_cols(qa.qxs, rp)), "xsq"
            assert np.array_equal(res["xss"].view(np.float32)[:M].view(np.uint32), qa.sxs.view(np.uint32)), "sxs"
        return
    xq = res["xq"][: M * K // 2].reshape(M, K // 2)
    assert np.array_equal(xq, O.pack_nibbles(qa.qx)), f"xq mismatch at {np.argwhere(xq != O.pack_nibbles(qa.qx))[:5]}"
    if qa.fmt == "int4":
        assert np.array_equal(res["xs"].view(np.float32)[:M].view(np.uint32), qa.sx.view(np.uint32)), "sx"
        if r > 0:
            xsq = res["xsq"][: M * rp // 2].reshape(M, rp // 2)
            assert np.array_equal(xsq, O.pack_nibbles(pad_cols(qa.qxs, rp))), "xsq"
            assert np.array_equal(res["xss"].view(np.float32)[:M].view(np.uint32), qa.sxs.view(np.uint32)), "sxs"
    else:
        assert np.array_equal(atoms_to_rows(res["xs"], M, K // 32), O.e8m0(qa.Ex)), "x E8M0"
        if r > 0:
            xsq = res["xsq"][: M * rp // 2].reshape(M, rp // 2)
            assert np.array_equal(xsq, O.pack_nibbles(pad_cols(qa.qxs, rp))), "xsq"
            assert np.array_equal(atoms_to_rows(res["xss"], M, rp // 32),
                                  O.e8m0(pad_cols(qa.Exs, rp // 32, fill=-127))), "xs E8M0"


def compare_y(Y_gpu: np.ndarray, Y_ref: np.ndarray, tol: float = YTOL):
    norms = np.linalg.norm(Y_ref, axis=1)
    err = np.abs(Y_gpu.astype(np.float64) - Y_ref).max(axis=1)
    zero = norms == 0
    assert np.all(Y_gpu[zero] == 0), "zero rows must give exact zeros"
    rel = err[~zero] / norms[~zero]
    worst = float(rel.max(initial=0.0))
    assert worst <= tol, f"max row-normalised error {worst:.3e} > {tol}"
    return worst


def oracle_host_parts(prep: O.Prepared) -> dict:
    """The oracle's prepared weight in the canonical host form of a checkpoint
    (serq_weight_host): row-major E8M0 bytes, residual padded to rp."""
    r, rp = prep.r, rp_of(prep.r)
    N, K = prep.qw.shape
    parts = {"perm": prep.perm.astype(np.int32), "s": prep.s.astype(np.float32),
             "inv_s": prep.inv_s.astype(np.float32), "wq": O.pack_nibbles(prep.qw)}
    if prep.fmt in O.INT_WEIGHT_FORMATS:
        parts["w_scale"] = prep.sw.astype(np.float32)
        parts["r_scale"] = prep.sR.astype(np.float32) if r > 0 else np.zeros(N, np.float32)
        parts["rq"] = O.pack_nibbles(pad_cols(prep.qR, rp)) if r > 0 else np.zeros((N, 0), np.uint8)
    else:
        parts["w_scale"] = O.e8m0(prep.Ew)
        if r > 0:
            parts["rq"] = O.pack_nibbles(pad_cols(prep.qR, rp))
            parts["r_scale"] = O.e8m0(pad_cols(prep.ER, rp // 32, fill=-127))
        else:
            parts["rq"] = np.zeros((N, 0), np.uint8)
            parts["r_scale"] = np.zeros((N, 0), np.uint8)
    return {k: np.ascontiguousarray(v) for k, v in parts.items()}


def assert_parts_equal(a: dict, b: dict):
    for k in ("perm", "s", "inv_s", "wq", "w_scale", "rq", "r_scale"):
        x, y = np.ascontiguousarray(a[k]), np.ascontiguousarray(b[k])
        assert x.nbytes == y.nbytes, (k, x.shape, y.shape)
        assert np.array_equal(x.view(np.uint8).reshape(-1), y.view(np.uint8).reshape(-1)), k
