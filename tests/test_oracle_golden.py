"""The oracle still reproduces its stored values on the tiny fp32 workload."""
import json
import os

import numpy as np

from golden.make_golden import OUT, TIMES, compute


def test_oracle_matches_golden():
    doc = json.load(open(OUT))
    assert doc["times"] == TIMES
    _, out = compute()
    np.testing.assert_allclose(out["y"][0, TIMES], np.array(doc["y_at_times"]), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(out["h_final"][0], np.array(doc["h_final"]), rtol=1e-12, atol=1e-14)
    fro = [float(np.linalg.norm(out["h_ckpt"][0, k])) for k in range(out["h_ckpt"].shape[1])]
    np.testing.assert_allclose(fro, doc["h_ckpt_fro"], rtol=1e-12)
    np.testing.assert_allclose(float(out["v"].astype(np.float64).sum()), doc["v_sum"], rtol=1e-12)
    np.testing.assert_array_equal(out["tail_out"][0], np.array(doc["tail_out"], dtype=np.float32))
