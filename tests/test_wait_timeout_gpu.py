"""The bounded pipeline wait on a GPU: a wait that nothing completes runs out
after its short limit, is reported as SERQ_ETIMEOUT by serq_device_status,
and leaves the context usable (no trap, no hang)."""

import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


def test_completed_wait_reports_ok(lib):
    import w4a4_post_quantization_serq_b200 as S
    S.serq_device_status()
    S.serq_selftest_wait(2_000_000, arrive=True)
    S.serq_device_status()


def test_wait_that_runs_out_reports_timeout(lib):
    import w4a4_post_quantization_serq_b200 as S
    S.serq_device_status()
    S.serq_selftest_wait(2_000_000, arrive=False)  # ~1 ms at boost clock
    with pytest.raises(S.SerqError) as e:
        S.serq_device_status()
    assert e.value.status == 5  # SERQ_ETIMEOUT
    assert "0xf01" in str(e.value)
    S.serq_device_status()  # the record was cleared
    # the context still computes
    x = torch.arange(16, device="cuda", dtype=torch.float32)
    assert float((x * 2).sum().item()) == 240.0


def test_limit_is_validated(lib):
    import w4a4_post_quantization_serq_b200 as S
    for bad in (0, -5, 5_000_000_000):
        with pytest.raises(S.SerqError):
            S.serq_selftest_wait(bad, arrive=True)
