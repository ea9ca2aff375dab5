"""GPU decode step (ssd_decode_step) against the CPU oracle.

One decode step is the layer on a one-token segment, so the reference is the
oracle's layer run over the same tokens: single steps from random and from
empty (state, conv tail), long runs of steps updated in place, and a decode
run that continues a prefix processed by ssd_stream_forward.
"""
import numpy as np
import pytest
import torch

import mamba_selective_state_causal_b200 as ssd
import oracle
import ssd_synth
from parity_util import TOL, host, rel_l2

pytestmark = pytest.mark.gpu
W = ssd_synth.WORKLOADS


def _inputs(wl, seed=0):
    prm = ssd_synth.make_params(wl, seed=seed)
    u = ssd_synth.make_u(wl, seed=seed)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"], seed=seed)
    return prm, u, dt


def _oracle(wl, u, prm, dt, tail=None, h0=None):
    io = "bf16" if wl.dtype == "bf16" else "f32"
    return oracle.layer(host(u), prm["w"].numpy(), host(dt), prm["A"].numpy(), prm["D"].numpy(),
                        prm["bias"].numpy(), None if tail is None else host(tail),
                        None if h0 is None else host(h0).astype(np.float64),
                        H=wl.H, P=wl.P, N=wl.N, G=wl.G, s=0, io_round=io)


def _decode_run(wl, u, prm, dt, tail=None, h0=None):
    """Run ssd_decode_step over every token of u, state and tail updated in place."""
    d = "cuda"
    g = {k: v.to(d) for k, v in prm.items()}
    ud, dtd = u.to(d), dt.to(d)
    h = (torch.zeros(wl.b, wl.H, wl.P, wl.N, device=d) if h0 is None else h0.to(d).clone())
    tl = (torch.zeros(wl.b, 3, wl.cch, dtype=u.dtype, device=d) if tail is None else tail.to(d).clone())
    ys = []
    for t in range(u.shape[1]):
        out = ssd.decode_step(ud[:, t].contiguous(), g["w"], dtd[:, t].contiguous(), g["A"], g["D"],
                              H=wl.H, P=wl.P, N=wl.N, G=wl.G, conv_bias=g["bias"],
                              tail_in=tl, tail_out=tl, h_in=h, h_out=h)
        ys.append(out["y"].clone())
    ssd.sync_status()
    return torch.stack(ys, 1), h, tl


@pytest.mark.parametrize("wl", [
    ssd_synth.scaled(W[1], L=1, b=3),                                  # 0.3B head shape, bf16
    ssd_synth.scaled(W[0], L=1, b=2, H=4, P=16, N=32, G=2),            # fp32, two groups
], ids=lambda w: f"{w.dtype}-b{w.b}-H{w.H}-P{w.P}-N{w.N}-G{w.G}")
def test_single_step_matches_oracle(wl):
    prm, u, dt = _inputs(wl)
    tail = ssd_synth.make_tail(wl)
    h0 = ssd_synth.make_h0(wl, scale=0.5)
    d = "cuda"
    g = {k: v.to(d) for k, v in prm.items()}
    out = ssd.decode_step(u[:, 0].contiguous().to(d), g["w"], dt[:, 0].contiguous().to(d), g["A"], g["D"],
                          H=wl.H, P=wl.P, N=wl.N, G=wl.G, conv_bias=g["bias"], tail_in=tail.to(d),
                          h_in=h0.to(d))
    ssd.sync_status()
    ref = _oracle(wl, u, prm, dt, tail=tail, h0=h0)
    tol = TOL[wl.dtype]
    assert rel_l2(host(out["y"]).reshape(wl.b, 1, -1), ref["y"].reshape(wl.b, 1, -1)) <= tol
    assert rel_l2(host(out["h_out"]), ref["h_final"]) <= tol
    np.testing.assert_array_equal(host(out["tail_out"]), ref["tail_out"])


def test_first_token_from_empty_state():
    """NULL tail_in and h_in mean zeros, as at the start of a stream."""
    wl = ssd_synth.scaled(W[1], L=1, b=2, H=4)
    prm, u, dt = _inputs(wl, seed=3)
    d = "cuda"
    g = {k: v.to(d) for k, v in prm.items()}
    out = ssd.decode_step(u[:, 0].contiguous().to(d), g["w"], dt[:, 0].contiguous().to(d), g["A"], g["D"],
                          H=wl.H, P=wl.P, N=wl.N, conv_bias=g["bias"])
    ssd.sync_status()
    ref = _oracle(wl, u, prm, dt)
    assert rel_l2(host(out["y"]).reshape(wl.b, 1, -1), ref["y"].reshape(wl.b, 1, -1)) <= TOL["bf16"]
    assert rel_l2(host(out["h_out"]), ref["h_final"]) <= TOL["bf16"]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_steps_in_place_equal_one_segment(dtype):
    """48 decode steps, state and tail updated in place, against the layer over the 48 tokens."""
    base = W[1] if dtype == "bf16" else W[0]
    wl = ssd_synth.scaled(base, L=48, b=2, H=4, P=64 if dtype == "bf16" else 16,
                          N=128 if dtype == "bf16" else 16)
    prm, u, dt = _inputs(wl, seed=5)
    tail = ssd_synth.make_tail(wl)
    h0 = ssd_synth.make_h0(wl, scale=0.5)
    y, h, tl = _decode_run(wl, u, prm, dt, tail=tail, h0=h0)
    ref = _oracle(wl, u, prm, dt, tail=tail, h0=h0)
    tol = TOL[dtype]
    assert rel_l2(host(y).reshape(wl.b, wl.L, -1), ref["y"].reshape(wl.b, wl.L, -1)) <= tol
    assert rel_l2(host(h), ref["h_final"]) <= tol
    np.testing.assert_array_equal(host(tl), ref["tail_out"])


def test_decode_continues_a_streamed_prefix():
    """ssd_stream_forward over 512 tokens, then 16 decode steps from its (h_final, tail_out)."""
    wl = ssd_synth.scaled(W[1], L=528, b=1, H=4)
    prm, u, dt = _inputs(wl, seed=7)
    d = "cuda"
    g = {k: v.to(d) for k, v in prm.items()}
    pre = ssd.stream_forward(u[:, :512].contiguous().to(d), g["w"], dt[:, :512].contiguous().to(d), g["A"],
                             g["D"], H=wl.H, P=wl.P, N=wl.N, Q=wl.Q, s=0, conv_bias=g["bias"])
    sub = ssd_synth.scaled(wl, L=16)
    y, h, tl = _decode_run(sub, u[:, 512:].contiguous(), prm, dt[:, 512:].contiguous(),
                           tail=pre["tail_out"].cpu(), h0=pre["h_final"].cpu())
    ref = _oracle(wl, u, prm, dt)
    got_y = np.concatenate([host(pre["y"]).reshape(1, 512, -1), host(y).reshape(1, 16, -1)], 1)
    assert rel_l2(got_y, ref["y"].reshape(1, 528, -1)) <= TOL["bf16"]
    assert rel_l2(host(h), ref["h_final"]) <= TOL["bf16"]
    np.testing.assert_array_equal(host(tl), ref["tail_out"])


def test_bench_configuration_256_streams():
    """The configuration the decode bench times: 256 independent streams of the 0.3B shape (32 heads
    of P = 64, N = 128, 2304 conv channels, bf16), each from an empty state and conv tail, eight
    steps with the state and tail updated in place and y written into the caller's buffer; every
    step's y and the final state against the oracle's layer over the eight tokens of each stream,
    the conv tail bitwise."""
    wl = ssd_synth.scaled(W[1], b=256, L=8, segments=1)
    prm, u, dt = _inputs(wl, seed=21)
    d = "cuda"
    g = {k: v.to(d) for k, v in prm.items()}
    u_steps = u.to(d).transpose(0, 1).contiguous()
    dt_steps = dt.to(d).transpose(0, 1).contiguous()
    h = torch.zeros(wl.b, wl.H, wl.P, wl.N, device=d)
    tl = torch.zeros(wl.b, 3, wl.cch, dtype=u.dtype, device=d)
    y = torch.empty(wl.b, wl.H, wl.P, dtype=u.dtype, device=d)
    ys = []
    for t in range(wl.L):
        ssd.decode_step(u_steps[t], g["w"], dt_steps[t], g["A"], g["D"], H=wl.H, P=wl.P, N=wl.N, G=wl.G,
                        conv_bias=g["bias"], tail_in=tl, tail_out=tl, h_in=h, h_out=h, y=y)
        ys.append(y.clone())
    ssd.sync_status()
    ref = _oracle(wl, u, prm, dt)
    got = host(torch.stack(ys, 1)).reshape(wl.b, wl.L, -1)
    want = ref["y"].reshape(wl.b, wl.L, -1)
    for t in range(wl.L):
        assert rel_l2(got[:, t], want[:, t]) <= TOL["bf16"], t
    assert rel_l2(host(h), ref["h_final"]) <= TOL["bf16"]
    np.testing.assert_array_equal(host(tl), ref["tail_out"])
