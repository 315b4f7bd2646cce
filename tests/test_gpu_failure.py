"""The failure path on the GPU, without a fault: a bounded wait that runs
out is reported through the device error word, the word is cleared once
read, and the context keeps running kernels correctly afterwards."""
import pytest

import oracle
import workloads as wl
from gpu_common import TOL_F32, rel_err, run_scan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hm():
    import torch
    assert torch.cuda.is_available()
    import selective_ssm_sequence_b200 as mod
    return mod


def test_bounded_wait_reports_timeout_and_context_survives(hm):
    assert hm.hm_get_device_error() == hm.HM_OK
    hm.hm_selftest_wait_timeout(4096)
    assert hm.hm_get_device_error() == hm.HM_ERR_TIMEOUT
    assert "kernel id 10" in hm.lib.hm_last_error_detail().decode()
    # read once, then cleared
    assert hm.hm_get_device_error() == hm.HM_OK
    # the context still computes: the tiny fp32 scan against the oracle
    inp = wl.scan_inputs(wl.TINY_F32)
    o, _, _ = run_scan(hm, inp, "f32")
    ref = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], W_q=inp["W_q"], W_k=inp["W_k"])
    assert rel_err(o, ref) <= TOL_F32


def test_selftest_rejects_bad_poll_counts(hm):
    with pytest.raises(hm.HMError):
        hm.hm_selftest_wait_timeout(0)
    with pytest.raises(hm.HMError):
        hm.hm_selftest_wait_timeout(1 << 21)
    assert hm.hm_get_device_error() == hm.HM_OK
