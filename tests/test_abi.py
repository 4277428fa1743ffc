"""The C ABI library: loads, exports every declared symbol, validates arguments.

CPU-only: no call here reaches a kernel (argument checks run before any
device access).
"""

import ctypes

import pytest

from w4a4_post_quantization_serq_b200 import _native as N


def test_library_exports_every_header_function(lib):
    names = N.header_functions()
    assert len(names) >= 10
    for name in names:
        assert hasattr(lib, name), name


def test_version_string(lib):
    assert b"sm_100a" in lib.serq_version()


@pytest.mark.parametrize("M,K,r,fmt", [(2048, 4096, 128, 0), (1, 14336, 16, 1), (77, 256, 0, 1), (64, 256, 256, 0)])
def test_act_buffer_sizes_closed_form(lib, M, K, r, fmt):
    sz = N.ActSizes()
    assert lib.serq_act_buffer_sizes(M, K, r, fmt, ctypes.byref(sz)) == N.SERQ_OK
    rp = ((r + 63) // 64) * 64 if r else 0
    assert sz.xq == M * K // 2 and sz.xsq == M * rp // 2
    if fmt == 0:
        assert sz.xs == 4 * M and sz.xss == (4 * M if r else 0)
    else:
        rb = (M + 127) // 128
        assert sz.xs == rb * (K // 128) * 512
        assert sz.xss == (rb * ((rp // 32 + 3) // 4) * 512 if r else 0)


@pytest.mark.parametrize("M,K,r,fmt", [(0, 256, 0, 0), (4, 200, 0, 0), (4, 256, -1, 0), (4, 256, 300, 1),
                                       (4, 256, 0, 7)])
def test_act_buffer_sizes_rejects(lib, M, K, r, fmt):
    sz = N.ActSizes()
    assert lib.serq_act_buffer_sizes(M, K, r, fmt, ctypes.byref(sz)) == N.SERQ_EINVAL
    assert lib.serq_last_error()


def test_quant_act_rejects_before_touching_device(lib):
    # NULL buffers and unaligned pointers are refused with EINVAL
    assert lib.serq_quant_act(None, 4, 256, 0, 0, None, None, None, None, None) == N.SERQ_EINVAL
    assert lib.serq_quant_act(16, 4, 256, 16, 0, 32, 48, None, None, None) == N.SERQ_EINVAL  # r>0 w/o slice bufs
    assert lib.serq_quant_act(17, 4, 256, 0, 0, 32, 48, None, None, None) == N.SERQ_EINVAL  # unaligned


def test_prepare_rejects_bad_descriptors(lib):
    h = ctypes.c_void_p()
    for K, Nn, r, fmt, W, a, s in [(200, 256, 0, 0, 16, 16, None), (256, 100, 0, 0, 16, 16, None),
                                    (256, 256, 257, 0, 16, 16, None), (256, 256, 0, 3, 16, 16, None),
                                    (256, 256, 0, 0, 16, None, None), (256, 256, 0, 0, 16, 16, 32),
                                    (256, 256, 0, 0, 17, 16, None), (256, 256, 0, 0, None, 16, None)]:
        desc = N.PrepareDesc(K, Nn, r, fmt, W, a, s)
        assert lib.serq_prepare(ctypes.byref(desc), ctypes.byref(h), None) == N.SERQ_EINVAL, (K, Nn, r, fmt)
        assert h.value is None


def test_linear_rejects_null_weight(lib):
    assert lib.serq_linear(None, 4, 16, 16, None, None, 16, None, None) == N.SERQ_EINVAL


def test_selftest_wait_rejects_bad_limits(lib):
    for bad in (0, -1, 4_000_000_001):
        assert lib.serq_selftest_wait(bad, 1, None) == N.SERQ_EINVAL
        assert b"limit_cycles" in lib.serq_last_error()


def test_calib_absmax_rejects_before_touching_device(lib):
    assert lib.serq_calib_absmax(None, 4, 256, 16, None) == N.SERQ_EINVAL   # NULL X
    assert lib.serq_calib_absmax(16, 0, 256, 16, None) == N.SERQ_EINVAL     # M < 1
    assert lib.serq_calib_absmax(16, 4, 0, 16, None) == N.SERQ_EINVAL       # K < 1
    assert lib.serq_calib_absmax(17, 4, 256, 16, None) == N.SERQ_EINVAL     # unaligned


def test_view_and_fold_reject_null_weight(lib):
    view = N.WeightView()
    assert lib.serq_weight_get_view(None, ctypes.byref(view)) == N.SERQ_EINVAL
    assert lib.serq_fold_producer(None, 16, 4, 32, None) == N.SERQ_EINVAL


@pytest.mark.parametrize("M,K,Nn,r", [(0, 256, 256, 0), (17, 256, 256, 0), (4, 200, 256, 0), (4, 256, 200, 0),
                                      (4, 65536, 256, 0), (4, 256, 256, 257), (4, 256, 256, -1)])
def test_noalloc_rejects_bad_shapes(lib, M, K, Nn, r):
    assert lib.serq_linear_small_m_noalloc(M, K, Nn, r, 16, 16, 16, 16, 16, 16, 16, 16, 16, None) == N.SERQ_EINVAL
    assert lib.serq_last_error()


def test_noalloc_rejects_null_and_unaligned(lib):
    ok = (4, 256, 256, 16)
    # NULL weight codes
    assert lib.serq_linear_small_m_noalloc(*ok, None, 16, 16, 16, 16, 16, 16, 16, 16, None) == N.SERQ_EINVAL
    # r > 0 without the residual / salient-slice buffers
    assert lib.serq_linear_small_m_noalloc(*ok, 16, 16, None, 16, 16, 16, 16, 16, 16, None) == N.SERQ_EINVAL
    # an unaligned output pointer
    assert lib.serq_linear_small_m_noalloc(*ok, 16, 16, 16, 16, 16, 16, 16, 16, 24, None) == N.SERQ_EINVAL


def test_block_entry_points_reject_before_touching_device(lib):
    # RoPE: NULL / unaligned x, odd head_dim, ld narrower than the heads, base <= 1
    assert lib.serq_rope(None, 4, 256, 2, 128, ctypes.c_float(10000.0), 0, None) == N.SERQ_EINVAL
    assert lib.serq_rope(18, 4, 256, 2, 128, ctypes.c_float(10000.0), 0, None) == N.SERQ_EINVAL
    assert lib.serq_rope(16, 4, 256, 2, 127, ctypes.c_float(10000.0), 0, None) == N.SERQ_EINVAL
    assert lib.serq_rope(16, 4, 200, 2, 128, ctypes.c_float(10000.0), 0, None) == N.SERQ_EINVAL
    assert lib.serq_rope(16, 4, 256, 2, 128, ctypes.c_float(1.0), 0, None) == N.SERQ_EINVAL
    # attention: NULL, head_dim other than 128, heads not grouping, short leading dims, unaligned
    att = lib.serq_attention_prefill
    assert att(None, 256, 16, 16, 128, 4, 2, 1, 128, 16, 256, None) == N.SERQ_EINVAL
    assert att(16, 128, 16, 16, 64, 4, 2, 1, 64, 16, 128, None) == N.SERQ_EUNSUPPORTED
    assert att(16, 384, 16, 16, 256, 4, 3, 2, 128, 16, 384, None) == N.SERQ_EINVAL
    assert att(16, 128, 16, 16, 128, 4, 2, 1, 128, 16, 256, None) == N.SERQ_EINVAL
    assert att(24, 256, 16, 16, 128, 4, 2, 1, 128, 16, 256, None) == N.SERQ_EINVAL
    # add: n not a multiple of 8, NULL, unaligned
    assert lib.serq_add(16, 16, 16, 12, None) == N.SERQ_EINVAL
    assert lib.serq_add(None, 16, 16, 16, None) == N.SERQ_EINVAL
    assert lib.serq_add(16, 20, 16, 16, None) == N.SERQ_EINVAL
