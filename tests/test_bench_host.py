"""Host-side logic of bench.py, on CPU: the multi-rank plumbing under gloo
(world size 2) and the reference arm's JSON line (the oracle on a tiny
workload).  No GPU: the linear itself is covered by the parity tests."""

from __future__ import annotations

import io
import json
import os
import socket
import subprocess
import sys
import types
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

_RANK_SCRIPT = r"""
import io, json, os, sys, types
from contextlib import redirect_stdout
sys.path.insert(0, os.getcwd())
import bench
world, rank, local, pg = bench.dist_setup(2)
assert pg is not None
bench.barrier(pg)
t = bench.max_over_ranks(pg, 10.0 + 5.0 * rank)          # per-rank step time (ms)
v = bench.whole_job_tops(world, 1e12, t)                  # every rank runs 1e12 flops per step
buf = io.StringIO()
args = types.SimpleNamespace(cpu_rows=4, steps=1, warmup=0)
if rank != 0:
    with redirect_stdout(buf):
        bench.reference_main(args, world, rank, pg)       # non-zero ranks exit without work
bench.barrier(pg)
pg.destroy_process_group()
print(json.dumps({"rank": rank, "world": world, "local": local, "max_ms": t, "tops": v,
                  "ref_out": buf.getvalue()}))
"""


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_gloo_two_ranks_host_logic():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2",
                   RANK=str(rank), LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", _RANK_SCRIPT], cwd=ROOT, env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=180)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            pytest.fail("gloo ranks did not finish")
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for rank, o in enumerate(outs):
        assert o["rank"] == rank and o["world"] == 2 and o["local"] == rank
        assert o["max_ms"] == 15.0                       # max over ranks, the same on every rank
        assert o["tops"] == pytest.approx(2 * 1e12 / 15e-3 / 1e12)
    assert outs[1]["ref_out"] == ""                      # only rank 0 prints the reference line


def test_whole_job_is_replica_sum():
    one = bench.whole_job_tops(1, 3e12, 2.0)
    assert bench.whole_job_tops(8, 3e12, 2.0) == pytest.approx(8 * one)
    assert one == pytest.approx(3e12 / 2e-3 / 1e12)


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(None, 3.5) == 3.5


def test_reference_arm_json_line(monkeypatch):
    """--impl reference: the oracle on a row sample; one JSON line with the contract's keys."""
    monkeypatch.setattr(bench, "WORKLOAD", "tiny_int4")
    args = types.SimpleNamespace(cpu_rows=8, steps=2, warmup=1)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.reference_main(args, 1, 0, None)
    lines = [l for l in buf.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["n_gpus"] == 1
    assert line["value"] > 0 and line["unit"] == "TOPS" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "TOPS", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    # rank 1 of a multi-rank launch prints nothing
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.reference_main(args, 2, 1, None)
    assert buf.getvalue() == ""


def test_captured_traffic_tracks_source(tmp_path, monkeypatch):
    """The committed DRAM traffic is reported only for the kernel source it was measured on."""
    rec = json.load(open(bench.CAPTURED_TRAFFIC_FILE))
    fake = dict(rec, source_sha256_prefix="0" * 16)
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps(fake))
    monkeypatch.setattr(bench, "CAPTURED_TRAFFIC_FILE", str(p))
    assert bench.captured_traffic() is None
    fake = dict(rec, kernel="some_other_kernel")
    p.write_text(json.dumps(fake))
    assert bench.captured_traffic() is None


def test_quant_act_bytes_closed_form():
    # LLaMA-3-8B down input, M=2048, K=14336, r=128 (rp=128), MXFP4: read X^ 58.7 MB,
    # write codes 14.7 MB + 0.13 MB and E8M0 scales 0.92 MB + 8 KB
    import bench
    M, K = 2048, 14336
    assert bench.quant_act_bytes(M, K, 128, "mxfp4") == 2 * M * K + M * K // 2 + M * 64 + M * K // 32 + M * 4
    # INT4, LLaMA-2-7B q_proj: fp32 per-token scales for the row and the slice
    assert bench.quant_act_bytes(2048, 4096, 128, "int4") == 2 * 2048 * 4096 + 2048 * 2048 + 2048 * 64 + 8 * 2048
    assert bench.quant_act_bytes(16, 4096, 0, "int4") == 2 * 16 * 4096 + 16 * 2048 + 4 * 16


def test_quant_act_bytes_w4a8():
    import bench
    assert bench.quant_act_bytes(2048, 4096, 128, "w4a8") == 2 * 2048 * 4096 + 2048 * 4096 + 2048 * 128 + 8 * 2048
