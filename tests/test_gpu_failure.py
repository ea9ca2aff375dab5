"""Failure detection without a GPU fault: a bounded wait is made to run out.

The test hook SSD_TEST_DROP_UNIT makes one CTA's producer skip its loads in the
first scan call of a process, so the consumers of that CTA wait on a barrier
that nothing completes.  Every wait in the tensor-core kernels is bounded
(SSD_WAIT_LIMIT_MS): the CTA must give up, drain its MMAs, free its TMEM and
latch SSD_ERR_TIMEOUT in the device status word, which ssd_sync_status()
reports.  The context must stay usable: the next call computes the right
answer.  The library reads its hooks once per process, so the case runs in a
child process that starts with them set.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def _child():
    sys.path.insert(0, HERE)
    sys.path.insert(0, os.path.dirname(HERE))
    import mamba_selective_state_causal_b200 as ssd
    import ssd_synth
    from parity_util import TOL, check_outputs
    from test_gpu_scan import run_case

    wl = ssd_synth.scaled(ssd_synth.WORKLOADS[1], L=2048, H=4)
    try:
        run_case(wl)          # run_case ends with sync_status()
    except ssd.SSDError as err:
        assert err.code == 8, err
    else:
        raise AssertionError("the dropped unit did not time out")
    ssd.sync_status()         # the status word was cleared by the failing read
    out, ref = run_case(wl)   # and the context still computes correct results
    check_outputs(out, ref, TOL["bf16"])
    print("child ok")


@pytest.mark.gpu
def test_wait_that_runs_out_reports_timeout():
    env = dict(os.environ, SSD_TEST_DROP_UNIT="0", SSD_WAIT_LIMIT_MS="200")
    r = subprocess.run([sys.executable, os.path.abspath(__file__)], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "child ok" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]


if __name__ == "__main__":
    _child()
