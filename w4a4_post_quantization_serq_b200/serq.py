"""Python binding of the SERQ C ABI: same names as include/serq.h.

Argument marshalling only. Device buffers are torch CUDA tensors, the stream
is torch's current stream, and every computation runs in libserq.so's CUDA
kernels. There is no CPU path: calls fail when the library is not built or
no sm_100 device is present.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np
import torch

from . import _native as N


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return t.data_ptr()


def _fmt(fmt) -> int:
    return N.FMT[fmt] if isinstance(fmt, str) else int(fmt)


class _DeviceView:
    """Zero-copy torch view of library-owned device memory."""

    def __init__(self, ptr: int, shape, typestr: str, owner):
        self.owner = owner
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (ptr, False),
                                         "version": 3, "strides": None}


def _view(ptr, shape, typestr, owner) -> torch.Tensor:
    return torch.as_tensor(_DeviceView(ptr, shape, typestr, owner), device="cuda")


class SerqWeight:
    """A prepared SERQ linear (owns its device buffers through the library)."""

    def __init__(self, handle: int, K: int, N_: int, r: int, fmt: int):
        self.handle = ctypes.c_void_p(handle)
        self.K, self.N, self.r, self.fmt = K, N_, r, fmt
        self.rp = ((r + 63) // 64) * 64 if r > 0 else 0

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            try:
                N.load().serq_weight_destroy(h)
            except Exception:  # interpreter shutdown: the library may already be gone
                pass
            self.handle = None

    def view(self) -> Dict[str, torch.Tensor]:
        """Device tensors of perm, s, inv_s, packed W^_q / Q(R) and their scales."""
        return serq_weight_get_view(self)


def serq_calib_absmax(X: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M, K = X.shape
    if out is None:
        out = torch.empty(K, dtype=torch.float32, device=X.device)
    N.check(N.load().serq_calib_absmax(_ptr(X), M, K, _ptr(out), _stream(stream)))
    return out


def serq_prepare(W: torch.Tensor, r: int, fmt, act_absmax: Optional[torch.Tensor] = None,
                 s: Optional[torch.Tensor] = None, R: Optional[torch.Tensor] = None, stream=None) -> SerqWeight:
    """Offline preparation of one linear; W is bf16 K x N (Y = X W). Synchronizes.

    R (bf16 r x N, optional) fills the residual slot with a given matrix (the
    second factor of the two-factor baseline) instead of W~_s - Q(W~_s)."""
    if W.dtype != torch.bfloat16:
        raise ValueError("W must be bfloat16")
    K, N_ = W.shape
    desc = N.PrepareDesc(K, N_, r, _fmt(fmt), _ptr(W), _ptr(act_absmax), _ptr(s), _ptr(R))
    h = ctypes.c_void_p()
    N.check(N.load().serq_prepare(ctypes.byref(desc), ctypes.byref(h), _stream(stream)))
    return SerqWeight(h.value, K, N_, r, _fmt(fmt))


def serq_weight_get_view(w: SerqWeight) -> Dict[str, torch.Tensor]:
    v = N.WeightView()
    N.check(N.load().serq_weight_get_view(w.handle, ctypes.byref(v)))
    out = {
        "perm": _view(v.perm, (v.K,), "<i4", w),
        "s": _view(v.s, (v.K,), "<f4", w),
        "inv_s": _view(v.inv_s, (v.K,), "<f4", w),
        "wq": _view(v.wq, (v.N, v.K // 2), "|u1", w),
    }
    if v.fmt != N.FMT["mxfp4"]:  # INT4 weights (W4A4, W4A8): fp32 per-channel scales
        out["w_scale"] = _view(v.w_scale, (v.N,), "<f4", w)
        if v.rp > 0:
            out["rq"] = _view(v.rq, (v.N, v.rp // 2), "|u1", w)
            out["r_scale"] = _view(v.r_scale, (v.N,), "<f4", w)
    else:
        out["w_scale"] = _view(v.w_scale, (v.w_scale_bytes,), "|u1", w)
        if v.rp > 0:
            out["rq"] = _view(v.rq, (v.N, v.rp // 2), "|u1", w)
            out["r_scale"] = _view(v.r_scale, (v.r_scale_bytes,), "|u1", w)
    return out


def _host_parts(K: int, N_: int, r: int, rp: int, fmt: int) -> Dict[str, np.ndarray]:
    """Zeroed numpy buffers of the canonical host form (see serq_weight_host in serq.h)."""
    out = {"perm": np.zeros(K, np.int32), "s": np.zeros(K, np.float32), "inv_s": np.zeros(K, np.float32),
           "wq": np.zeros((N_, K // 2), np.uint8), "rq": np.zeros((N_, rp // 2), np.uint8)}
    if fmt != N.FMT["mxfp4"]:
        out["w_scale"] = np.zeros(N_, np.float32)
        out["r_scale"] = np.zeros(N_, np.float32)
    else:
        out["w_scale"] = np.zeros((N_, K // 32), np.uint8)
        out["r_scale"] = np.zeros((N_, rp // 32), np.uint8)
    return out


def _host_struct(parts: Dict[str, np.ndarray], K: int, N_: int, r: int, rp: int, fmt: int):
    """serq_weight_host pointing into contiguous numpy arrays (kept alive by the caller)."""
    def p(name):
        a = parts.get(name)
        if a is None or a.size == 0:
            return None
        if not a.flags["C_CONTIGUOUS"]:
            raise ValueError(f"{name} must be C-contiguous")
        return a.ctypes.data
    return N.WeightHost(K, N_, r, rp, fmt, p("perm"), p("s"), p("inv_s"), p("wq"), p("w_scale"), p("rq"),
                        p("r_scale"))


def serq_weight_export(w: SerqWeight) -> Dict[str, np.ndarray]:
    """Canonical host copies of a prepared weight (perm, s, inv_s, wq, w_scale, rq, r_scale)."""
    parts = _host_parts(w.K, w.N, w.r, w.rp, w.fmt)
    st = _host_struct(parts, w.K, w.N, w.r, w.rp, w.fmt)
    N.check(N.load().serq_weight_export(w.handle, ctypes.byref(st)))
    return parts


def serq_weight_create_from_host(parts: Dict[str, np.ndarray], K: int, N_: int, r: int, fmt,
                                 stream=None) -> SerqWeight:
    """A prepared weight on the current device from canonical host arrays. Synchronizes."""
    f = _fmt(fmt)
    rp = ((r + 63) // 64) * 64 if r > 0 else 0
    keep = {k: np.ascontiguousarray(v) for k, v in parts.items() if v is not None}
    st = _host_struct(keep, K, N_, r, rp, f)
    h = ctypes.c_void_p()
    N.check(N.load().serq_weight_create_from_host(ctypes.byref(st), ctypes.byref(h), _stream(stream)))
    return SerqWeight(h.value, K, N_, r, f)


def serq_weight_save(w: SerqWeight, path: str) -> None:
    N.check(N.load().serq_weight_save(w.handle, os.fsencode(path)))


def serq_weight_load(path: str, stream=None) -> SerqWeight:
    h = ctypes.c_void_p()
    N.check(N.load().serq_weight_load(os.fsencode(path), ctypes.byref(h), _stream(stream)))
    info = N.WeightHost()
    N.check(N.load().serq_weight_export(h, ctypes.byref(info)))
    return SerqWeight(h.value, info.K, info.N, info.r, info.fmt)


def serq_weight_file_write(path: str, parts: Dict[str, np.ndarray], K: int, N_: int, r: int, fmt) -> None:
    """Write a checkpoint from canonical host arrays (no GPU needed)."""
    f = _fmt(fmt)
    rp = ((r + 63) // 64) * 64 if r > 0 else 0
    keep = {k: np.ascontiguousarray(v) for k, v in parts.items() if v is not None}
    st = _host_struct(keep, K, N_, r, rp, f)
    N.check(N.load().serq_weight_file_write(os.fsencode(path), ctypes.byref(st)))


def serq_weight_file_read(path: str):
    """Read a checkpoint into canonical host arrays (no GPU needed): (parts, K, N, r, fmt)."""
    info = N.WeightHost()
    N.check(N.load().serq_weight_file_read(os.fsencode(path), ctypes.byref(info)))
    parts = _host_parts(info.K, info.N, info.r, info.rp, info.fmt)
    st = _host_struct(parts, info.K, info.N, info.r, info.rp, info.fmt)
    N.check(N.load().serq_weight_file_read(os.fsencode(path), ctypes.byref(st)))
    return parts, info.K, info.N, info.r, info.fmt


def serq_debug_fail_next_allocations(n: int) -> int:
    """Test hook: the next n weight allocations fail with SERQ_ENOMEM (no cudaMalloc)."""
    return int(N.load().serq_debug_fail_next_allocations(int(n)))


def serq_fold_producer(w: SerqWeight, src: torch.Tensor, dst: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """dst[row, i] = bf16(src[row, perm[i]] / s[perm[i]])."""
    rows = src.shape[0]
    if dst is None:
        dst = torch.empty_like(src)
    N.check(N.load().serq_fold_producer(w.handle, _ptr(src), rows, _ptr(dst), _stream(stream)))
    return dst


def serq_act_buffer_sizes(M: int, K: int, r: int, fmt) -> Dict[str, int]:
    sz = N.ActSizes()
    N.check(N.load().serq_act_buffer_sizes(M, K, r, _fmt(fmt), ctypes.byref(sz)))
    return {"xq": sz.xq, "xs": sz.xs, "xsq": sz.xsq, "xss": sz.xss}


@dataclass
class QuantAct:
    M: int
    K: int
    r: int
    fmt: int
    xq: torch.Tensor
    xs: torch.Tensor
    xsq: Optional[torch.Tensor]
    xss: Optional[torch.Tensor]


def alloc_act(M: int, K: int, r: int, fmt, device="cuda") -> QuantAct:
    sz = serq_act_buffer_sizes(M, K, r, fmt)

    def buf(n):
        return torch.empty(max(n, 16), dtype=torch.uint8, device=device) if n > 0 else None
    return QuantAct(M, K, r, _fmt(fmt), buf(sz["xq"]), buf(sz["xs"]), buf(sz["xsq"]), buf(sz["xss"]))


def serq_quant_act(Xhat: torch.Tensor, r: int, fmt, out: Optional[QuantAct] = None, stream=None) -> QuantAct:
    """Per-token INT4 / MXFP4 quantization of X^ and of its salient slice X^[:, :r]."""
    M, K = Xhat.shape
    if out is None:
        out = alloc_act(M, K, r, fmt, Xhat.device)
    N.check(N.load().serq_quant_act(_ptr(Xhat), M, K, r, _fmt(fmt), _ptr(out.xq), _ptr(out.xs), _ptr(out.xsq),
                                    _ptr(out.xss), _stream(stream)))
    return out


def serq_rmsnorm_quant_act(w: SerqWeight, H: torch.Tensor, gamma: torch.Tensor, eps: float,
                           out: Optional[QuantAct] = None, xhat: Optional[torch.Tensor] = None,
                           stream=None) -> QuantAct:
    """RMSNorm producer with w's fold and the activation quantization in one pass (H: bf16 M x K)."""
    M = H.shape[0]
    if out is None:
        out = alloc_act(M, w.K, w.r, w.fmt, H.device)
    N.check(N.load().serq_rmsnorm_quant_act(w.handle, _ptr(H), _ptr(gamma), float(eps), M, _ptr(out.xq),
                                            _ptr(out.xs), _ptr(out.xsq), _ptr(out.xss), _ptr(xhat),
                                            _stream(stream)))
    return out


def serq_swiglu_quant_act(w: SerqWeight, Ygu: torch.Tensor, out: Optional[QuantAct] = None,
                          xhat: Optional[torch.Tensor] = None, stream=None) -> QuantAct:
    """SwiGLU producer ([gate | up], bf16 M x 2K) with w's fold and the quantization in one pass."""
    M = Ygu.shape[0]
    if out is None:
        out = alloc_act(M, w.K, w.r, w.fmt, Ygu.device)
    N.check(N.load().serq_swiglu_quant_act(w.handle, _ptr(Ygu), M, _ptr(out.xq), _ptr(out.xs), _ptr(out.xsq),
                                           _ptr(out.xss), _ptr(xhat), _stream(stream)))
    return out


def serq_fold_quant_act(w: SerqWeight, X: torch.Tensor, out: Optional[QuantAct] = None,
                        xhat: Optional[torch.Tensor] = None, stream=None) -> QuantAct:
    """serq_fold_producer's fold and serq_quant_act in one pass (X: bf16 M x K)."""
    M = X.shape[0]
    if out is None:
        out = alloc_act(M, w.K, w.r, w.fmt, X.device)
    N.check(N.load().serq_fold_quant_act(w.handle, _ptr(X), M, _ptr(out.xq), _ptr(out.xs), _ptr(out.xsq),
                                         _ptr(out.xss), _ptr(xhat), _stream(stream)))
    return out


def _strided_ptr(t: torch.Tensor) -> int:
    """Pointer of a 2-D CUDA tensor whose rows are contiguous (a column slice of a row-major matrix)."""
    if not t.is_cuda or t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D CUDA tensor with contiguous rows")
    return t.data_ptr()


def serq_rope(x: torch.Tensor, n_heads: int, head_dim: int, base: float, pos0: int = 0, stream=None) -> torch.Tensor:
    """In-place rotate-half RoPE on the first n_heads heads of x (bf16 [M, >= n_heads*head_dim], rows contiguous)."""
    N.check(N.load().serq_rope(_strided_ptr(x), x.shape[0], x.stride(0), n_heads, head_dim, float(base), pos0,
                               _stream(stream)))
    return x


def serq_attention_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_q: int, n_kv: int,
                           out: Optional[torch.Tensor] = None, head_dim: int = 128, stream=None) -> torch.Tensor:
    """Causal grouped-query attention (bf16; q, k, v may be column slices of one QKV matrix)."""
    M = q.shape[0]
    if out is None:
        out = torch.empty(M, n_q * head_dim, dtype=torch.bfloat16, device=q.device)
    N.check(N.load().serq_attention_prefill(_strided_ptr(q), q.stride(0), _strided_ptr(k), _strided_ptr(v), k.stride(0),
                                            M, n_q, n_kv, head_dim, _strided_ptr(out), out.stride(0),
                                            _stream(stream)))
    return out


def serq_add(a: torch.Tensor, b: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out = bf16(a + b) elementwise."""
    if out is None:
        out = torch.empty_like(a)
    N.check(N.load().serq_add(_ptr(a), _ptr(b), _ptr(out), a.numel(), _stream(stream)))
    return out


def serq_linear(w: SerqWeight, qa: QuantAct, Y: Optional[torch.Tensor] = None,
                acc_dbg: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y = X^_q W^_q + X~_{s,q} Q(R), bf16 M x N, in one kernel launch."""
    if Y is None:
        Y = torch.empty(qa.M, w.N, dtype=torch.bfloat16, device=qa.xq.device)
    N.check(N.load().serq_linear(w.handle, qa.M, _ptr(qa.xq), _ptr(qa.xs), _ptr(qa.xsq), _ptr(qa.xss), _ptr(Y),
                                 _ptr(acc_dbg), _stream(stream)))
    return Y


def serq_prepare_swiglu(W_gate_up: torch.Tensor, r: int, down: SerqWeight, act_absmax: Optional[torch.Tensor] = None,
                        s: Optional[torch.Tensor] = None, stream=None) -> SerqWeight:
    """The gate/up linear ([W_gate | W_up], bf16 K x 2F) with down's permutation folded into its output
    columns, for serq_linear_swiglu_quant. Synchronizes."""
    K, N_ = W_gate_up.shape
    desc = N.PrepareDesc(K, N_, r, N.FMT["mxfp4"], _ptr(W_gate_up), _ptr(act_absmax), _ptr(s), None)
    h = ctypes.c_void_p()
    N.check(N.load().serq_prepare_swiglu(ctypes.byref(desc), down.handle, ctypes.byref(h), _stream(stream)))
    w = SerqWeight(h.value, K, N_, r, N.FMT["mxfp4"])
    w.down = down
    return w


def serq_linear_swiglu_quant(w: SerqWeight, qa: QuantAct, out: Optional[QuantAct] = None,
                             xhat: Optional[torch.Tensor] = None, stream=None) -> QuantAct:
    """gate/up linear whose epilogue writes down's quantized input (SiLU(gate) * up, folded 1/s)."""
    F = w.N // 2
    if out is None:
        out = alloc_act(qa.M, F, w.down.r, "mxfp4", qa.xq.device)
    N.check(N.load().serq_linear_swiglu_quant(w.handle, qa.M, _ptr(qa.xq), _ptr(qa.xs), _ptr(qa.xsq), _ptr(qa.xss),
                                              _ptr(out.xq), _ptr(out.xs), _ptr(out.xsq), _ptr(out.xss), _ptr(xhat),
                                              _stream(stream)))
    return out


def serq_linear_l2qer(main: SerqWeight, l1: SerqWeight, qa: QuantAct, Y: Optional[torch.Tensor] = None,
                      scratch: Optional[dict] = None, stream=None) -> torch.Tensor:
    """Two-factor baseline Y = X_q W_q + Q(X_q L1_q) L2_q (three launches; see serq.h)."""
    M, k = qa.M, main.r
    if scratch is None:
        scratch = {"T": torch.empty(M, k, dtype=torch.bfloat16, device=qa.xq.device),
                   "tq": alloc_act(M, k, k, main.fmt, qa.xq.device)}
    if Y is None:
        Y = torch.empty(M, main.N, dtype=torch.bfloat16, device=qa.xq.device)
    t = scratch["tq"]
    N.check(N.load().serq_linear_l2qer(main.handle, l1.handle, M, _ptr(qa.xq), _ptr(qa.xs), _ptr(scratch["T"]),
                                       _ptr(t.xq), _ptr(t.xs), _ptr(t.xsq), _ptr(t.xss), _ptr(Y), _stream(stream)))
    return Y


def serq_linear_small_m_noalloc(M: int, K: int, N_: int, r: int, wq: torch.Tensor, w_scale: torch.Tensor,
                                rq: Optional[torch.Tensor], r_scale: Optional[torch.Tensor], qa: QuantAct,
                                Y: torch.Tensor, stream=None) -> torch.Tensor:
    """Small-M MXFP4 linear from caller-owned buffers only; the library allocates nothing.

    For callers that cannot allocate device memory on their serving path: the
    split-K scratch lives in a static device array of the library (calls that
    overlap on the GPU race on it). Output Y must be preallocated (bf16 M x N).
    """
    N.check(N.load().serq_linear_small_m_noalloc(M, K, N_, r, _ptr(wq), _ptr(w_scale), _ptr(rq), _ptr(r_scale),
                                                 _ptr(qa.xq), _ptr(qa.xs), _ptr(qa.xsq), _ptr(qa.xss), _ptr(Y),
                                                 _stream(stream)))
    return Y


def serq_device_status(stream=None) -> None:
    """Synchronize and raise SerqError(SERQ_ETIMEOUT) if a kernel wait timed out."""
    N.check(N.load().serq_device_status(_stream(stream)))


def serq_selftest_wait(limit_cycles: int, arrive: bool, stream=None) -> None:
    """Launch the bounded-wait self-test kernel (see include/serq.h)."""
    N.check(N.load().serq_selftest_wait(int(limit_cycles), 1 if arrive else 0, _stream(stream)))


def serq_version() -> str:
    return N.load().serq_version().decode()
