"""A prepared weight as an artefact, on the GPU: export, checkpoint, import.

* serq_prepare's device weight, exported to the canonical host form, equals
  the oracle's preparation bit for bit;
* serq_weight_save writes the same bytes as a checkpoint written from the
  oracle's preparation;
* serq_weight_load and serq_weight_create_from_host give weights whose
  serq_linear matches the oracle (bit-exact INT4 accumulators, bf16 Y within
  2e-3 of the row norm);
* the out-of-memory path returns SERQ_ENOMEM and leaks no device memory.
(SERQ reading notes Stage 3, gist.science/zh 2.3: the folded, permuted and
quantized linear is produced offline and reused.)
"""

import numpy as np
import pytest
import torch

import w4a4_post_quantization_serq_b200 as S
from oracle import serq_oracle as O
from synth import activations, weights
from w4a4_post_quantization_serq_b200 import _native as NAT

from parity_util import assert_parts_equal, compare_y, oracle_host_parts, to_dev_bf16

pytestmark = pytest.mark.gpu

CASES = [("int4", 64, 512, 384, 128), ("int4", 33, 256, 256, 0), ("mxfp4", 300, 512, 640, 40),
         ("mxfp4", 4, 1024, 512, 128), ("mxfp4", 64, 256, 256, 256)]


def _problem(M, K, N, seed=7):
    X = activations(seed, M, K, max(1, K // 100), "lognormal", 50.0)
    W = weights(seed + 1, K, N)
    return X, W


def _linear_vs_oracle(w, X, prep, fmt, r):
    M = X.shape[0]
    Xh = S.serq_fold_producer(w, to_dev_bf16(X))
    qa = S.serq_quant_act(Xh, r, fmt)
    acc = torch.zeros(2, M, w.N, dtype=torch.int32, device="cuda") if fmt == "int4" else None
    Y = S.serq_linear(w, qa, acc_dbg=acc)
    S.serq_device_status()
    ref = O.linear(prep, O.quant_act(O.fold_activation(X, prep.s, prep.perm), r, fmt))
    if fmt == "int4":
        a = acc.cpu().numpy()
        assert np.array_equal(a[0], ref.acc1) and np.array_equal(a[1], ref.acc2)
    return compare_y(Y.float().cpu().numpy(), ref.Y)


@pytest.mark.parametrize("fmt,M,K,N,r", CASES)
def test_export_save_load_create(tmp_path, fmt, M, K, N, r):
    X, W = _problem(M, K, N)
    a = O.calib_absmax(X)
    prep = O.prepare(W, r, fmt, act_absmax=a)
    parts = oracle_host_parts(prep)

    w = S.serq_prepare(to_dev_bf16(W), r, fmt, act_absmax=torch.from_numpy(a).cuda())
    assert_parts_equal(S.serq_weight_export(w), parts)

    # checkpoint written from the device weight == checkpoint written from the oracle
    p_dev, p_ora = str(tmp_path / "dev.serq"), str(tmp_path / "ora.serq")
    S.serq_weight_save(w, p_dev)
    S.serq_weight_file_write(p_ora, parts, K, N, r, fmt)
    assert open(p_dev, "rb").read() == open(p_ora, "rb").read()

    # a loaded weight and one built from the oracle's host arrays compute the same linear
    wl = S.serq_weight_load(p_ora)
    assert (wl.K, wl.N, wl.r, wl.fmt) == (K, N, r, NAT.FMT[fmt])
    assert_parts_equal(S.serq_weight_export(wl), parts)
    _linear_vs_oracle(wl, X, prep, fmt, r)
    wc = S.serq_weight_create_from_host(parts, K, N, r, fmt)
    _linear_vs_oracle(wc, X, prep, fmt, r)
    # and so does the weight prepared on the device
    _linear_vs_oracle(w, X, prep, fmt, r)


def test_out_of_memory_path_leaks_nothing(tmp_path):
    K, N, r, fmt = 512, 512, 64, "mxfp4"
    X, W = _problem(16, K, N)
    Wd = to_dev_bf16(W)
    a = S.serq_calib_absmax(to_dev_bf16(X))
    ok = S.serq_prepare(Wd, r, fmt, act_absmax=a)
    path = str(tmp_path / "w.serq")
    S.serq_weight_save(ok, path)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    S.serq_debug_fail_next_allocations(3)
    for call in (lambda: S.serq_prepare(Wd, r, fmt, act_absmax=a), lambda: S.serq_weight_load(path),
                 lambda: S.serq_weight_create_from_host(S.serq_weight_export(ok), K, N, r, fmt)):
        with pytest.raises(S.SerqError) as e:
            call()
        assert e.value.status == NAT.SERQ_ENOMEM
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    assert S.serq_debug_fail_next_allocations(0) == 0
    # the library still works afterwards
    again = S.serq_prepare(Wd, r, fmt, act_absmax=a)
    assert_parts_equal(S.serq_weight_export(again), S.serq_weight_export(ok))
