"""Whole layer (conv1d+SiLU then scan, ssd_stream_forward) against the CPU oracle.

Covers the workloads of the benchmark table: the tiny fp32 case and the
0.3B L=16k case in full; the 0.3B 1M-token stream as 8 resumed segments,
the 1.3B b=2 L=256k and the 2.7B b=4 L=64k shapes at full size, with the
oracle run on sampled heads over the whole sequence (it cannot afford all
heads at 1M tokens); and the split/resume invariant with its negative control.
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


def gpu_layer(wl, u, prm, dt, segments=1, h0=None, tail=None, zero_tail_at=None, fused=False, two_call=False):
    """Run the layer on the GPU as `segments` consecutive resumed calls of ssd_stream_forward
    (on the tensor-core shapes the conv of x runs inside the scan's first pass); fused=True
    asks for no conv output (v in the workspace); two_call=True uses ssd_conv_forward then
    ssd_scan_forward instead (one conv kernel over every channel)."""
    d = "cuda"
    g = {k: v.to(d) for k, v in prm.items()}
    L = u.shape[1]
    seg = L // segments
    st = None if h0 is None else h0.to(d).clone()
    tl = None if tail is None else tail.to(d).clone()
    ys, cks = [], []
    if fused:
        code = ssd.SSD_BF16 if wl.dtype == "bf16" else ssd.SSD_F32
        ws = torch.empty(max(1, ssd.stream_workspace_size(wl.b, seg, wl.H, wl.P, wl.N, wl.G, wl.Q, code)),
                         dtype=torch.uint8, device=d)
    else:
        ws = ssd.alloc_workspace(wl.b, seg, wl.H, wl.P, wl.N, wl.Q, d)
    for k in range(segments):
        sl = slice(k * seg, (k + 1) * seg if k < segments - 1 else L)
        if zero_tail_at is not None and k == zero_tail_at:
            tl = torch.zeros_like(tl)
        if two_call:
            to = torch.empty(wl.b, 3, wl.cch, dtype=u.dtype, device=d)
            v, _ = ssd.conv_forward(u[:, sl], g["w"], g["bias"], tail_in=tl, tail_out=to)
            di, gn = wl.H * wl.P, wl.G * wl.N
            y, hf, hc = ssd.scan_forward(v[:, :, :di], v[:, :, di:di + gn], v[:, :, di + gn:], dt[:, sl], g["A"],
                                         g["D"], st, H=wl.H, G=wl.G, Q=wl.Q, s=wl.s)
            out = {"y": y, "h_final": hf, "h_ckpt": hc, "tail_out": to}
        else:
            out = ssd.stream_forward(u[:, sl], g["w"], dt[:, sl], g["A"], g["D"], H=wl.H, P=wl.P,
                                     N=wl.N, G=wl.G, Q=wl.Q, s=wl.s, conv_bias=g["bias"], tail_in=tl,
                                     h0=st, workspace=ws if sl.stop - sl.start == seg else None,
                                     keep_v=not fused)
        st, tl = out["h_final"], out["tail_out"]
        ys.append(out["y"])
        if out["h_ckpt"] is not None:
            cks.append(out["h_ckpt"])
    ssd.sync_status()
    return {"y": torch.cat(ys, 1), "h_final": st, "tail_out": tl,
            "h_ckpt": torch.cat(cks, 1) if cks else None}


def oracle_layer(wl, u, prm, dt, heads=None, h0=None, tail=None):
    """Oracle on the whole sequence; with `heads`, only the channels those heads read."""
    u = u if isinstance(u, np.ndarray) else host(u)
    w = prm["w"].numpy()
    bias = prm["bias"].numpy()
    A, D = prm["A"].numpy(), prm["D"].numpy()
    dtn = dt if isinstance(dt, np.ndarray) else host(dt)
    io = "bf16" if wl.dtype == "bf16" else "f32"
    if heads is None:
        return oracle.layer(u, w, dtn, A, D, bias, None if tail is None else host(tail),
                            None if h0 is None else host(h0).astype(np.float64),
                            H=wl.H, P=wl.P, N=wl.N, G=wl.G, s=wl.s, io_round=io)
    di = wl.H * wl.P
    cols = np.concatenate([np.arange(h * wl.P, (h + 1) * wl.P) for h in heads] +
                          [np.arange(di, di + 2 * wl.N)])
    sub = ssd_synth.scaled(wl, H=len(heads))
    return oracle.layer(u[:, :, cols] if u.shape[2] != len(cols) else u, w[cols], dtn[:, :, heads],
                        A[heads], D[heads], bias[cols], None, None, H=len(heads), P=wl.P, N=wl.N,
                        G=1, s=wl.s, io_round=io)


FUSED = pytest.mark.parametrize("fused", [False, True], ids=["v_returned", "v_in_workspace"])


@FUSED
def test_tiny_f32_workload(fused):
    wl = W[0]
    prm = ssd_synth.make_params(wl)
    u = ssd_synth.make_u(wl)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"])
    out = gpu_layer(wl, u.cuda(), prm, dt.cuda(), fused=fused)
    ref = oracle_layer(wl, u, prm, dt)
    check_outputs(out, ref, TOL["f32"])
    np.testing.assert_array_equal(host(out["tail_out"]), ref["tail_out"])


@FUSED
def test_03b_L16k_workload_all_heads(fused):
    wl = W[1]
    prm = ssd_synth.make_params(wl)
    u = ssd_synth.make_u(wl)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"])
    out = gpu_layer(wl, u.cuda(), prm, dt.cuda(), fused=fused)
    ref = oracle_layer(wl, u, prm, dt)
    errs = check_outputs(out, ref, TOL["bf16"])
    print("0.3B L16k relL2", errs)


@FUSED
@pytest.mark.parametrize("segments", [2, 8])
def test_streamed_segments_equal_unsplit(segments, fused):
    """Split/resume invariant: consecutive resumed calls reproduce the unsplit layer."""
    wl = ssd_synth.scaled(W[2], L=8 * 2048, H=4, s=1024)
    prm = ssd_synth.make_params(wl)
    u = ssd_synth.make_u(wl)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"])
    h0 = ssd_synth.make_h0(wl, scale=0.5)
    tail = ssd_synth.make_tail(wl)
    out = gpu_layer(wl, u.cuda(), prm, dt.cuda(), segments=segments, h0=h0, tail=tail, fused=fused)
    ref = oracle_layer(wl, u, prm, dt, h0=h0, tail=tail)
    check_outputs(out, ref, TOL["bf16"])
    np.testing.assert_array_equal(host(out["tail_out"]), ref["tail_out"])
    one = gpu_layer(wl, u.cuda(), prm, dt.cuda(), segments=1, h0=h0, tail=tail, fused=fused)
    assert rel_l2(host(out["y"]), host(one["y"])) < 1e-2


@FUSED
def test_resume_without_conv_tail_differs(fused):
    """Negative control: resuming with a zero conv buffer changes the output."""
    wl = ssd_synth.scaled(W[2], L=4 * 512, H=2)
    prm = ssd_synth.make_params(wl)
    u = ssd_synth.make_u(wl)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"])
    good = gpu_layer(wl, u.cuda(), prm, dt.cuda(), segments=4, tail=torch.zeros(1, 3, wl.cch).to(torch.bfloat16),
                     fused=fused)
    bad = gpu_layer(wl, u.cuda(), prm, dt.cuda(), segments=4, tail=torch.zeros(1, 3, wl.cch).to(torch.bfloat16),
                    zero_tail_at=2, fused=fused)
    ref = oracle_layer(wl, u, prm, dt)
    check_outputs(good, ref, TOL["bf16"])
    yb = host(bad["y"])
    seg = wl.L // 4
    assert rel_l2(yb[:, 2 * seg:2 * seg + 3], ref["y"][:, 2 * seg:2 * seg + 3]) > 1e-2


def test_fused_conv_equals_two_call_path_bitwise():
    """The conv of x fused into the scan's first pass computes x exactly as the conv kernel
    does (same fused multiply-adds, same SiLU, same rounding), so ssd_stream_forward equals
    ssd_conv_forward followed by ssd_scan_forward bit for bit: several stripes, a ragged
    tail, a conv buffer and a state handed in, two batch rows."""
    wl = ssd_synth.scaled(W[1], L=3 * 2048 + 77, H=4, b=2, s=1024)
    prm = ssd_synth.make_params(wl)
    prm["bias"] = ssd_synth.make_conv_grads(wl)[1]
    u = ssd_synth.make_u(wl).cuda()
    dt = ssd_synth.make_dt(wl, prm["dt_bias"]).cuda()
    h0 = ssd_synth.make_h0(wl, scale=0.5)
    tail = ssd_synth.make_tail(wl)
    a = gpu_layer(wl, u, prm, dt, h0=h0, tail=tail, two_call=True)
    for fused in (False, True):
        b = gpu_layer(wl, u, prm, dt, h0=h0, tail=tail, fused=fused)
        for k in ("y", "h_final", "h_ckpt", "tail_out"):
            assert torch.equal(a[k], b[k]), (fused, k, rel_l2(host(a[k]), host(b[k])))


def _sampled_full_size(wl, heads, fused=True):
    prm = ssd_synth.make_params(wl)
    d = "cuda"
    u = ssd_synth.make_u(wl, device=d)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"].to(d), device=d)
    out = gpu_layer(wl, u, prm, dt, segments=wl.segments, fused=fused)
    di = wl.H * wl.P
    cols = torch.cat([torch.arange(h * wl.P, (h + 1) * wl.P) for h in heads] +
                     [torch.arange(di, di + 2 * wl.N)]).to(d)
    u_sub = host(u.index_select(2, cols))
    dt_h = host(dt)
    del u
    ref = oracle_layer(wl, u_sub, prm, dt_h, heads=heads)
    errs = check_outputs(out, ref, TOL["bf16"], heads=heads)
    print(wl.name, "sampled heads", heads, "relL2", errs)


@pytest.mark.slow
@FUSED
def test_03b_1M_stream_full_size_sampled_heads(fused):
    _sampled_full_size(W[2], heads=[0, 31], fused=fused)


@pytest.mark.slow
def test_13b_b2_L256k_full_size_sampled_heads():
    _sampled_full_size(W[3], heads=[5, 63])


@pytest.mark.slow
def test_27b_b4_L64k_full_size_sampled_heads():
    _sampled_full_size(W[4], heads=[0, 41, 79])
