"""serq_linear_small_m_noalloc: the small-M MXFP4 linear for callers that
cannot allocate device memory (its split-K scratch is a static device array
inside the library). Called through the C ABI and compared with serq_linear.

Kept in its own file, collected last, so that a run stopping at the first
failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from synth import activations, weights

pytestmark = pytest.mark.gpu

YTOL = 2e-3  # the GPU parity tests' output tolerance


def _rel_err(y, ref):
    y = y.float().cpu().numpy().astype(np.float64)
    ref = ref.float().cpu().numpy().astype(np.float64)
    norms = np.linalg.norm(ref, axis=1)
    assert np.all(norms > 0)
    return float((np.abs(y - ref).max(axis=1) / norms).max())


@pytest.mark.parametrize("M,K,N,r", [(1, 4096, 1024, 128), (16, 2048, 768, 40), (7, 512, 256, 0)])
def test_noalloc_matches_serq_linear_twice(lib, M, K, N, r):
    import w4a4_post_quantization_serq_b200 as S
    from w4a4_post_quantization_serq_b200 import _native as NV
    torch.cuda.set_device(0)
    X = torch.from_numpy(activations(500 + M, M, K, max(1, K // 100), "const", 50.0)).to(torch.bfloat16).cuda()
    Xc = torch.from_numpy(activations(600 + M, 256, K, max(1, K // 100), "const", 50.0)).to(torch.bfloat16).cuda()
    W = torch.from_numpy(weights(700 + K, K, N)).to(torch.bfloat16).cuda()
    w = S.serq_prepare(W, r, "mxfp4", act_absmax=S.serq_calib_absmax(Xc))
    qa = S.serq_quant_act(S.serq_fold_producer(w, X), r, "mxfp4")
    ref = S.serq_linear(w, qa)          # the existing entry point
    view = w.view()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def ptr(t):
        return None if t is None else t.data_ptr()

    outs = []
    for _ in range(2):                  # two calls in a row share the static scratch
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = lib.serq_linear_small_m_noalloc(M, K, N, r, ptr(view["wq"]), ptr(view["w_scale"]),
                                             ptr(view.get("rq")), ptr(view.get("r_scale")), ptr(qa.xq),
                                             ptr(qa.xs), ptr(qa.xsq), ptr(qa.xss), ptr(Y), stream)
        assert st == NV.SERQ_OK, lib.serq_last_error()
        outs.append(Y)
    assert lib.serq_device_status(stream) == NV.SERQ_OK
    for Y in outs:
        assert _rel_err(Y, ref) <= YTOL
        # both split reductions (static workspace here, cluster shared memory in
        # serq_linear) add the same partial sums in split order
        assert torch.equal(Y, ref)


def test_noalloc_rejects_sizes_beyond_the_static_scratch(lib):
    from w4a4_post_quantization_serq_b200 import _native as NV
    # 17 tokens (the small-M kernel takes at most 16)
    assert lib.serq_linear_small_m_noalloc(17, 256, 256, 0, 16, 16, None, None, 16, 16, None, None, 16,
                                           None) == NV.SERQ_EINVAL
    # M*N beyond the partial-sum area of the array
    assert lib.serq_linear_small_m_noalloc(16, 256, 65536 + 128 * 512, 0, 16, 16, None, None, 16, 16, None,
                                           None, 16, None) == NV.SERQ_EINVAL
    assert b"limit" in lib.serq_last_error()
