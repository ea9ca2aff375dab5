"""Failure detection without a GPU fault: a bounded wait is made to run out.

The test hook SSD_TEST_DROP_UNIT makes one CTA's producer skip its loads, so
the consumers of that CTA wait on a barrier that nothing completes.  Every
wait in the tensor-core kernels is bounded (SSD_WAIT_LIMIT_MS): the CTA must
give up, drain its MMAs, free its TMEM and latch SSD_ERR_TIMEOUT in the
device status word, which ssd_sync_status() reports.  The context must stay
usable: the next call computes the right answer.
"""
import pytest

import mamba_selective_state_causal_b200 as ssd
import ssd_synth
from parity_util import TOL, check_outputs
from test_gpu_scan import run_case

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_timeout(monkeypatch):
    wl = ssd_synth.scaled(ssd_synth.WORKLOADS[1], L=2048, H=4)
    monkeypatch.setenv("SSD_TEST_DROP_UNIT", "0")
    monkeypatch.setenv("SSD_WAIT_LIMIT_MS", "200")
    with pytest.raises(ssd.SSDError) as err:
        run_case(wl)          # run_case ends with sync_status()
    assert err.value.code == 8, err.value
    monkeypatch.delenv("SSD_TEST_DROP_UNIT")
    monkeypatch.delenv("SSD_WAIT_LIMIT_MS")
    ssd.sync_status()         # the status word was cleared by the failing read
    out, ref = run_case(wl)   # and the context still computes correct results
    check_outputs(out, ref, TOL["bf16"])
