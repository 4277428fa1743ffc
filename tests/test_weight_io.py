"""Checkpoint format of a prepared weight, through the C ABI without a GPU.

The weight is the oracle's preparation laid out in the canonical host form
(serq_weight_host); serq_weight_file_write / serq_weight_file_read must
round-trip it bit for bit and refuse damaged files and inconsistent content.
The offline artefact is the permuted, flattened, quantized linear (SERQ
reading notes Stage 3; gist.science/zh 2.3).
"""

import os
import struct

import numpy as np
import pytest

import w4a4_post_quantization_serq_b200 as S
from oracle import serq_oracle as O
from synth import activations, weights
from w4a4_post_quantization_serq_b200 import _native as NAT

from parity_util import assert_parts_equal, oracle_host_parts


def _prep(fmt, K, N, r, seed=5):
    X = activations(seed, 32, K, 3, "lognormal", 50.0)
    W = weights(seed + 1, K, N)
    return O.prepare(W, r, fmt, act_absmax=O.calib_absmax(X))


CASES = [("int4", 256, 128, 16), ("int4", 256, 256, 0), ("int4", 384, 128, 128),
         ("mxfp4", 256, 128, 16), ("mxfp4", 256, 256, 0), ("mxfp4", 512, 128, 40), ("mxfp4", 256, 128, 256)]


@pytest.mark.parametrize("fmt,K,N,r", CASES)
def test_file_round_trip_bit_exact(tmp_path, lib, fmt, K, N, r):
    prep = _prep(fmt, K, N, r)
    parts = oracle_host_parts(prep)
    path = str(tmp_path / "w.serq")
    S.serq_weight_file_write(path, parts, K, N, r, fmt)
    got, K2, N2, r2, fmt2 = S.serq_weight_file_read(path)
    assert (K2, N2, r2, fmt2) == (K, N, r, NAT.FMT[fmt])
    assert_parts_equal(got, parts)
    # header: magic, version, shape; then exactly the canonical payload
    raw = open(path, "rb").read()
    rp = ((r + 63) // 64) * 64 if r else 0
    assert raw[:8] == b"SERQWGT\0"
    version, f, k, n, rr, rpp, payload = struct.unpack_from("<I5iQ", raw, 8)
    assert (version, f, k, n, rr, rpp) == (1, NAT.FMT[fmt], K, N, r, rp)
    assert payload == sum(v.nbytes for v in parts.values()) and len(raw) == 64 + payload


def _written(tmp_path, fmt="mxfp4", K=256, N=128, r=16):
    prep = _prep(fmt, K, N, r)
    parts = oracle_host_parts(prep)
    path = str(tmp_path / "w.serq")
    S.serq_weight_file_write(path, parts, K, N, r, fmt)
    return path, parts


@pytest.mark.parametrize("damage", ["flip_payload", "truncate", "trailing", "magic", "version", "shape"])
def test_damaged_files_are_refused(tmp_path, lib, damage):
    path, _ = _written(tmp_path)
    raw = bytearray(open(path, "rb").read())
    if damage == "flip_payload":
        raw[64 + 1000] ^= 0x10
    elif damage == "truncate":
        raw = raw[:-7]
    elif damage == "trailing":
        raw += b"\0"
    elif damage == "magic":
        raw[0] = ord("X")
    elif damage == "version":
        raw[8] = 2
    elif damage == "shape":
        struct.pack_into("<i", raw, 16, 384)  # K
    open(path, "wb").write(bytes(raw))
    with pytest.raises(S.SerqError) as e:
        S.serq_weight_file_read(path)
    assert e.value.status == NAT.SERQ_EINVAL


def test_missing_file_is_refused(tmp_path, lib):
    with pytest.raises(S.SerqError) as e:
        S.serq_weight_file_read(str(tmp_path / "absent.serq"))
    assert e.value.status == NAT.SERQ_EINVAL


@pytest.mark.parametrize("fmt,bad", [
    ("int4", "perm_duplicate"), ("int4", "inv_s_ulp"), ("int4", "code_minus8"), ("int4", "s_zero"),
    ("int4", "code_past_r"), ("mxfp4", "e8m0_ff"), ("mxfp4", "r_scale_past_r"), ("mxfp4", "code_past_r"),
])
def test_inconsistent_content_is_refused(tmp_path, lib, fmt, bad):
    K, N, r = 256, 128, 16
    parts = oracle_host_parts(_prep(fmt, K, N, r))
    if bad == "perm_duplicate":
        parts["perm"][1] = parts["perm"][0]
    elif bad == "inv_s_ulp":
        parts["inv_s"][3] = np.nextafter(parts["inv_s"][3], np.float32(10))
    elif bad == "code_minus8":
        parts["wq"][5, 7] = (parts["wq"][5, 7] & 0xF0) | 0x8
    elif bad == "s_zero":
        parts["s"][2] = 0.0
    elif bad == "code_past_r":
        parts["rq"][0, r // 2] |= 0x01          # position r (first padded code)
    elif bad == "e8m0_ff":
        parts["w_scale"][3, 1] = 0xFF
    elif bad == "r_scale_past_r":
        parts["r_scale"][0, 1] = 120             # block 1 lies past r = 16
    with pytest.raises(S.SerqError) as e:
        S.serq_weight_file_write(str(tmp_path / "bad.serq"), parts, K, N, r, fmt)
    assert e.value.status == NAT.SERQ_EINVAL
    assert not os.path.exists(tmp_path / "bad.serq")


def test_null_arguments_are_refused(lib):
    assert lib.serq_weight_file_read(None, None) == NAT.SERQ_EINVAL
    assert lib.serq_weight_file_write(b"/nonexistent/x", None) == NAT.SERQ_EINVAL
    assert lib.serq_weight_save(None, b"x") == NAT.SERQ_EINVAL
    assert lib.serq_weight_export(None, None) == NAT.SERQ_EINVAL
    assert lib.serq_weight_create_from_host(None, None, None) == NAT.SERQ_EINVAL
    assert lib.serq_weight_load(None, None, None) == NAT.SERQ_EINVAL


def test_allocation_failure_hook_counts(lib):
    assert S.serq_debug_fail_next_allocations(3) == 0
    assert S.serq_debug_fail_next_allocations(0) == 3
