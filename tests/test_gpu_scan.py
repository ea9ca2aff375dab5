"""GPU selective scan (ssd_scan_forward) against the CPU oracle.

Sizes span several chunks, stripes and a ragged tail; edge cases cover L = 0,
L < Q, L an exact multiple of s (last checkpoint = final state), groups > 1,
long-dt decay underflow and the missing-D / missing-h0 variants.
"""
import numpy as np
import pytest
import torch

import mamba_selective_state_causal_b200 as ssd
import oracle
import ssd_synth
from parity_util import TOL, check_outputs, host, rel_l2

pytestmark = pytest.mark.gpu


def run_case(wl, seed=0, with_h0=True, with_D=True, dt_override=None, A_override=None):
    prm = ssd_synth.make_params(wl, seed=seed)
    x, Bm, Cm = ssd_synth.make_xbc(wl, seed=seed)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"], seed=seed) if dt_override is None else dt_override
    A = prm["A"] if A_override is None else A_override
    D = prm["D"] if with_D else None
    h0 = ssd_synth.make_h0(wl, seed=seed) if with_h0 else None
    d = "cuda"
    y, hf, hc = ssd.scan_forward(x.to(d), Bm.to(d), Cm.to(d), dt.to(d), A.to(d),
                                 None if D is None else D.to(d), None if h0 is None else h0.to(d),
                                 H=wl.H, G=wl.G, Q=wl.Q, s=wl.s)
    ssd.sync_status()
    ref = oracle.scan(x.float().numpy(), Bm.float().numpy(), Cm.float().numpy(), dt.numpy(),
                      A.numpy(), None if D is None else D.numpy(),
                      None if h0 is None else h0.double().numpy(), s=wl.s, H=wl.H, P=wl.P, G=wl.G)
    return {"y": y, "h_final": hf, "h_ckpt": hc}, ref


W = ssd_synth.WORKLOADS


@pytest.mark.parametrize("wl", [
    W[0],                                                                  # tiny fp32 workload
    ssd_synth.scaled(W[0], L=1000, b=2),                                   # several stripes, ragged
    ssd_synth.scaled(W[1], L=1000, H=4, b=2, s=256),                       # bf16, 0.3B head shape
    ssd_synth.scaled(W[1], L=777, H=3, P=32, N=64, Q=64, s=128),           # Q=64, odd H
    ssd_synth.scaled(W[1], L=300, H=2, P=16, N=32, Q=32, s=64),            # Q=32, bf16
    ssd_synth.scaled(W[0], L=500, H=4, G=2, P=32, N=32, Q=64, s=128),      # two groups, fp32
    ssd_synth.scaled(W[4], L=4096, H=6, b=2),                              # long dt: decay underflow
    ssd_synth.scaled(W[1], L=5000, H=5, P=128, N=16, Q=64, s=64, b=1),     # P=128, N=16
    ssd_synth.scaled(W[1], L=1500, H=8, G=2, b=1),                         # tensor cores, two B/C groups
], ids=lambda w: f"{w.dtype}-b{w.b}-L{w.L}-H{w.H}-P{w.P}-N{w.N}-G{w.G}-Q{w.Q}-s{w.s}")
def test_scan_matches_oracle(wl):
    out, ref = run_case(wl)
    check_outputs(out, ref, TOL[wl.dtype])


@pytest.mark.parametrize("L", [1, 31, 32, 64, 128, 129, 256])
def test_scan_short_sequences(L):
    wl = ssd_synth.scaled(W[0], L=L)
    out, ref = run_case(wl, seed=L)
    check_outputs(out, ref, TOL["f32"])
    if L % wl.s == 0:
        assert torch.equal(out["h_ckpt"][:, -1], out["h_final"])


def test_scan_without_D_and_h0():
    wl = ssd_synth.scaled(W[1], L=700, H=2)
    out, ref = run_case(wl, with_h0=False, with_D=False)
    check_outputs(out, ref, TOL["bf16"])


def test_scan_empty_sequence_returns_h0():
    wl = ssd_synth.scaled(W[1], L=0, H=2)
    h0 = ssd_synth.make_h0(wl).cuda()
    x = torch.empty(1, 0, wl.H * wl.P, dtype=torch.bfloat16, device="cuda")
    Bm = torch.empty(1, 0, wl.N, dtype=torch.bfloat16, device="cuda")
    dt = torch.empty(1, 0, wl.H, device="cuda")
    A = torch.full((wl.H,), -1.0, device="cuda")
    y, hf, _ = ssd.scan_forward(x, Bm, Bm, dt, A, None, h0, H=wl.H, Q=wl.Q, s=0)
    ssd.sync_status()
    assert torch.equal(hf, h0)


def test_scan_extreme_decay():
    """dt*A down to -8 per token: exp of large negative arguments underflows to 0."""
    wl = ssd_synth.scaled(W[4], L=600, H=3)
    dt = torch.full((wl.b, wl.L, wl.H), 0.5)
    A = torch.full((wl.H,), -16.0)
    out, ref = run_case(wl, dt_override=dt, A_override=A)
    check_outputs(out, ref, TOL["bf16"])
    assert torch.isfinite(out["y"].float()).all()


def test_scan_is_deterministic():
    wl = ssd_synth.scaled(W[1], L=3000, H=4)
    a, _ = run_case(wl)
    b, _ = run_case(wl)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_scan_linearity_in_h0():
    """y(h0_a + h0_b) - y(h0_b) is linear in h0 (x = 0 isolates the state term)."""
    wl = ssd_synth.scaled(W[0], L=400)
    prm = ssd_synth.make_params(wl)
    x, Bm, Cm = ssd_synth.make_xbc(wl)
    x = torch.zeros_like(x)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"])
    ha = ssd_synth.make_h0(wl, seed=1)
    d = "cuda"
    ya, _, _ = ssd.scan_forward(x.to(d), Bm.to(d), Cm.to(d), dt.to(d), prm["A"].to(d), None, ha.to(d),
                                H=wl.H, Q=wl.Q, s=0)
    y2, _, _ = ssd.scan_forward(x.to(d), Bm.to(d), Cm.to(d), dt.to(d), prm["A"].to(d), None,
                                (2 * ha).to(d), H=wl.H, Q=wl.Q, s=0)
    ssd.sync_status()
    assert rel_l2(host(y2), 2 * host(ya)) < 1e-6


def _generic_path_child(out_path):
    """Runs in a child process started with SSD_SCAN_PATH=generic (the library reads its
    hooks once per process): the CUDA-core scan of the same case, saved for the parent."""
    wl = ssd_synth.scaled(W[1], L=3000, H=4, b=2)
    slow, _ = run_case(wl)
    np.savez(out_path, **{k: host(v) for k, v in slow.items()})


def test_tensor_core_path_matches_cuda_core_path(tmp_path):
    """The tcgen05 path (bf16, P=64, N=128, Q=128) and the CUDA-core path agree,
    and both stay within tolerance of the oracle."""
    import os
    import subprocess
    import sys
    wl = ssd_synth.scaled(W[1], L=3000, H=4, b=2)
    fast, ref = run_case(wl)
    out = tmp_path / "generic.npz"
    here = os.path.dirname(os.path.abspath(__file__))
    code = (f"import sys; sys.path[:0] = [{here!r}, {os.path.dirname(here)!r}]; "
            f"import test_gpu_scan as t; t._generic_path_child({str(out)!r})")
    r = subprocess.run([sys.executable, "-c", code], env=dict(os.environ, SSD_SCAN_PATH="generic"),
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    slow = dict(np.load(out))
    check_outputs(fast, ref, TOL["bf16"])
    check_outputs({k: torch.from_numpy(v) for k, v in slow.items()}, ref, TOL["bf16"])
    assert rel_l2(host(fast["y"]), slow["y"]) < 1e-2
