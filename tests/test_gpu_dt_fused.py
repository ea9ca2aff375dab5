"""dt_bias + softplus + clamp fused into the kernels, against the oracle.

The entry points take the raw dt, its per-head bias, the softplus switch and
the clamp; the reference is the oracle run on oracle.dt_effective of the same
fp32 inputs.  Covers the tensor-core scan, the CUDA-core scan, a streamed
segment and the decode step.
"""
import numpy as np
import pytest
import torch

import mamba_selective_state_causal_b200 as ssd
import oracle
import ssd_synth
from parity_util import TOL, check_outputs, host, rel_l2

pytestmark = pytest.mark.gpu
W = ssd_synth.WORKLOADS


def _dt_inputs(wl, seed=0):
    prm = ssd_synth.make_params(wl, seed=seed)
    z = ssd_synth.make_dt_raw(wl, seed=seed)
    dt_eff = oracle.dt_effective(z.numpy(), prm["dt_bias"].numpy(), softplus=True, dt_min=wl.dt_min,
                                 dt_max=wl.dt_max)
    return prm, z, dt_eff


@pytest.mark.parametrize("wl", [
    ssd_synth.scaled(W[1], L=1000, H=4, b=2, s=256),          # tensor cores, bf16
    ssd_synth.scaled(W[0], L=500, H=4, G=2, P=32, N=32, Q=64, s=128),   # CUDA cores, fp32
], ids=lambda w: f"{w.dtype}-b{w.b}-L{w.L}-H{w.H}")
def test_scan_with_fused_dt(wl):
    prm, z, dt_eff = _dt_inputs(wl)
    x, Bm, Cm = ssd_synth.make_xbc(wl)
    h0 = ssd_synth.make_h0(wl)
    d = "cuda"
    y, hf, hc = ssd.scan_forward(x.to(d), Bm.to(d), Cm.to(d), z.to(d), prm["A"].to(d), prm["D"].to(d), h0.to(d),
                                 H=wl.H, G=wl.G, Q=wl.Q, s=wl.s, dt_bias=prm["dt_bias"].to(d), dt_softplus=True,
                                 dt_limit=(wl.dt_min, wl.dt_max))
    ssd.sync_status()
    ref = oracle.scan(x.float().numpy(), Bm.float().numpy(), Cm.float().numpy(), dt_eff, prm["A"].numpy(),
                      prm["D"].numpy(), h0.double().numpy(), s=wl.s, H=wl.H, P=wl.P, G=wl.G)
    check_outputs({"y": y, "h_final": hf, "h_ckpt": hc}, ref, TOL[wl.dtype])


def test_stream_segment_with_fused_dt():
    wl = ssd_synth.scaled(W[1], L=2048, H=4, s=1024)
    prm, z, dt_eff = _dt_inputs(wl, seed=2)
    u = ssd_synth.make_u(wl, seed=2)
    d = "cuda"
    g = {k: v.to(d) for k, v in prm.items()}
    out = ssd.stream_forward(u.to(d), g["w"], z.to(d), g["A"], g["D"], H=wl.H, P=wl.P, N=wl.N, Q=wl.Q, s=wl.s,
                             conv_bias=g["bias"], dt_bias=g["dt_bias"], dt_softplus=True,
                             dt_limit=(wl.dt_min, wl.dt_max))
    ssd.sync_status()
    ref = oracle.layer(u.float().numpy(), prm["w"].numpy(), dt_eff, prm["A"].numpy(), prm["D"].numpy(),
                       prm["bias"].numpy(), None, None, H=wl.H, P=wl.P, N=wl.N, G=wl.G, s=wl.s, io_round="bf16")
    check_outputs(out, ref, TOL["bf16"])


def test_decode_step_with_fused_dt():
    wl = ssd_synth.scaled(W[1], L=1, b=3, H=4)
    prm, z, dt_eff = _dt_inputs(wl, seed=4)
    u = ssd_synth.make_u(wl, seed=4)
    tail = ssd_synth.make_tail(wl)
    h0 = ssd_synth.make_h0(wl, scale=0.5)
    d = "cuda"
    g = {k: v.to(d) for k, v in prm.items()}
    out = ssd.decode_step(u[:, 0].contiguous().to(d), g["w"], z[:, 0].contiguous().to(d), g["A"], g["D"],
                          H=wl.H, P=wl.P, N=wl.N, conv_bias=g["bias"], tail_in=tail.to(d), h_in=h0.to(d),
                          dt_bias=g["dt_bias"], dt_softplus=True, dt_limit=(wl.dt_min, wl.dt_max))
    ssd.sync_status()
    ref = oracle.layer(u.float().numpy(), prm["w"].numpy(), dt_eff, prm["A"].numpy(), prm["D"].numpy(),
                       prm["bias"].numpy(), host(tail), host(h0).astype(np.float64), H=wl.H, P=wl.P, N=wl.N,
                       G=wl.G, s=0, io_round="bf16")
    assert rel_l2(host(out["y"]).reshape(wl.b, 1, -1), ref["y"].reshape(wl.b, 1, -1)) <= TOL["bf16"]
    assert rel_l2(host(out["h_out"]), ref["h_final"]) <= TOL["bf16"]
