"""ctypes declarations of the libserq.so C ABI (include/serq.h)."""

from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libserq.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "serq.h")

SERQ_OK, SERQ_EINVAL, SERQ_EUNSUPPORTED, SERQ_ENOMEM, SERQ_ECUDA, SERQ_ETIMEOUT = range(6)
FMT = {"int4": 0, "mxfp4": 1, "w4a8": 2}
STATUS_NAMES = {0: "SERQ_OK", 1: "SERQ_EINVAL", 2: "SERQ_EUNSUPPORTED", 3: "SERQ_ENOMEM",
                4: "SERQ_ECUDA", 5: "SERQ_ETIMEOUT"}

c_int, c_size_t, c_void_p, c_char_p = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_char_p


class PrepareDesc(ctypes.Structure):
    _fields_ = [("K", c_int), ("N", c_int), ("r", c_int), ("fmt", c_int),
                ("W", c_void_p), ("act_absmax", c_void_p), ("s", c_void_p), ("R", c_void_p)]


class WeightView(ctypes.Structure):
    _fields_ = [("K", c_int), ("N", c_int), ("r", c_int), ("rp", c_int), ("fmt", c_int),
                ("perm", c_void_p), ("s", c_void_p), ("inv_s", c_void_p),
                ("wq", c_void_p), ("wq_bytes", c_size_t),
                ("w_scale", c_void_p), ("w_scale_bytes", c_size_t),
                ("rq", c_void_p), ("rq_bytes", c_size_t),
                ("r_scale", c_void_p), ("r_scale_bytes", c_size_t)]


class WeightHost(ctypes.Structure):
    _fields_ = [("K", c_int), ("N", c_int), ("r", c_int), ("rp", c_int), ("fmt", c_int),
                ("perm", c_void_p), ("s", c_void_p), ("inv_s", c_void_p), ("wq", c_void_p),
                ("w_scale", c_void_p), ("rq", c_void_p), ("r_scale", c_void_p)]


class ActSizes(ctypes.Structure):
    _fields_ = [("xq", c_size_t), ("xs", c_size_t), ("xsq", c_size_t), ("xss", c_size_t)]


_SIGNATURES = {
    "serq_calib_absmax": (c_int, [c_void_p, c_int, c_int, c_void_p, c_void_p]),
    "serq_prepare": (c_int, [ctypes.POINTER(PrepareDesc), ctypes.POINTER(c_void_p), c_void_p]),
    "serq_weight_destroy": (None, [c_void_p]),
    "serq_weight_get_view": (c_int, [c_void_p, ctypes.POINTER(WeightView)]),
    "serq_fold_producer": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_void_p]),
    "serq_act_buffer_sizes": (c_int, [c_int, c_int, c_int, c_int, ctypes.POINTER(ActSizes)]),
    "serq_quant_act": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                               c_void_p]),
    "serq_rmsnorm_quant_act": (c_int, [c_void_p, c_void_p, c_void_p, ctypes.c_float, c_int, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_void_p]),
    "serq_swiglu_quant_act": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_void_p]),
    "serq_fold_quant_act": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_void_p]),
    "serq_rope": (c_int, [c_void_p, c_int, c_int, c_int, c_int, ctypes.c_float, c_int, c_void_p]),
    "serq_attention_prefill": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                                       c_void_p, c_int, c_void_p]),
    "serq_add": (c_int, [c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "serq_linear": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                            c_void_p]),
    "serq_prepare_swiglu": (c_int, [ctypes.POINTER(PrepareDesc), c_void_p, ctypes.POINTER(c_void_p), c_void_p]),
    "serq_linear_swiglu_quant": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "serq_linear_l2qer": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_void_p, c_void_p, c_void_p]),
    "serq_linear_small_m_noalloc": (c_int, [c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                            c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "serq_weight_export": (c_int, [c_void_p, ctypes.POINTER(WeightHost)]),
    "serq_weight_create_from_host": (c_int, [ctypes.POINTER(WeightHost), ctypes.POINTER(c_void_p), c_void_p]),
    "serq_weight_save": (c_int, [c_void_p, c_char_p]),
    "serq_weight_load": (c_int, [c_char_p, ctypes.POINTER(c_void_p), c_void_p]),
    "serq_weight_file_write": (c_int, [c_char_p, ctypes.POINTER(WeightHost)]),
    "serq_weight_file_read": (c_int, [c_char_p, ctypes.POINTER(WeightHost)]),
    "serq_debug_fail_next_allocations": (c_int, [c_int]),
    "serq_selftest_wait": (c_int, [ctypes.c_longlong, c_int, c_void_p]),
    "serq_device_status": (c_int, [c_void_p]),
    "serq_last_error": (c_char_p, []),
    "serq_version": (c_char_p, []),
}

_lib = None


def header_functions(path: str = HEADER):
    """Names of the functions include/serq.h declares."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(serq_[a-z0-9_]+)\s*\(", text)))


def load(path: str = LIB_PATH):
    """Load libserq.so once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with __graft_entry__.build() "
                           "or python -m w4a4_post_quantization_serq_b200.build")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class SerqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def check(status: int):
    if status != SERQ_OK:
        raise SerqError(status, (load().serq_last_error() or b"").decode())
