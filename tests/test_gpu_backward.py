"""GPU backward pass (ssd_scan_backward) against the CPU oracle's reverse mode.

The reference is always the oracle's full backpropagation (every state kept,
fp64).  The GPU recomputes each cell of s tokens from its checkpoint, as
MA-GC does on the sequence axis; the gradients must agree with plain
backpropagation to rel 1e-5 (the Video-Ma2mba verdict record,
skeptic_critique.concrete_test, asks exactly this of the cell recompute).
With exact checkpoints the GPU's fp32 arithmetic meets 1e-5 for bf16 inputs
too; with the checkpoints of the GPU's own bf16 forward the states carry
that forward's error, and the bf16 tolerance applies.
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
KEYS = ("dx", "dB", "dC", "ddt", "dA", "dD", "dh0")


def _inputs(wl, seed=0, h0=True):
    prm = ssd_synth.make_params(wl, seed=seed)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"], seed=seed)
    x, Bm, Cm = ssd_synth.make_xbc(wl, seed=seed)
    hz = ssd_synth.make_h0(wl, seed=seed) if h0 else None
    dy, dhf = ssd_synth.make_grads(wl, seed=seed)
    return prm, dt, x, Bm, Cm, hz, dy, dhf


def _oracle_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf):
    return oracle.scan_backward(x.float().numpy(), Bm.float().numpy(), Cm.float().numpy(), dt.numpy(),
                                prm["A"].numpy(), prm["D"].numpy(),
                                dy.float().numpy().reshape(wl.b, wl.L, wl.H, wl.P),
                                h0=None if h0 is None else h0.double().numpy(),
                                dh_final=None if dhf is None else dhf.double().numpy(),
                                H=wl.H, P=wl.P, G=wl.G)


def _gpu_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf, h_ckpt=None, s=0):
    d = "cuda"
    dev = lambda t: None if t is None else t.to(d)
    out = ssd.scan_backward(dev(x), dev(Bm), dev(Cm), dev(dt), dev(prm["A"]), dev(prm["D"]), dev(dy),
                            h0=dev(h0), h_ckpt=dev(h_ckpt), dh_final=dev(dhf), H=wl.H, G=wl.G, s=s)
    ssd.sync_status()
    return {k: host(v) for k, v in out.items()}


def _compare(got, ref, tol, wl):
    errs = {}
    for k in KEYS:
        g = got[k].reshape(ref[k].shape) if k != "dx" else got[k].reshape(wl.b, wl.L, wl.H, wl.P)
        errs[k] = rel_l2(g, ref[k])
    bad = {k: e for k, e in errs.items() if not e <= tol}
    assert not bad, f"relL2 above {tol}: {bad} (all: {errs})"


def test_cell_recompute_matches_full_backprop_fp32():
    """fp32, P = 64, L = 1024, s = 128: the checkpointed backward against full backprop."""
    wl = ssd_synth.scaled(W[0], b=2, L=1024, H=4, P=64, N=64, Q=64, s=128)
    prm, dt, x, Bm, Cm, h0, dy, dhf = _inputs(wl, seed=11)
    ref = _oracle_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf)
    fwd = ssd.scan_forward(x.cuda(), Bm.cuda(), Cm.cuda(), dt.cuda(), prm["A"].cuda(), prm["D"].cuda(),
                           h0.cuda(), H=wl.H, Q=wl.Q, s=wl.s)
    got = _gpu_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf, h_ckpt=fwd[2].cpu(), s=wl.s)
    _compare(got, ref, TOL["f32"], wl)


@pytest.mark.parametrize("L,s", [(1000, 256), (1024, 1024), (64, 64), (65, 64), (1, 64)])
def test_bf16_exact_checkpoints(L, s):
    """bf16 inputs at the 0.3B head shape, checkpoints from the oracle: the backward alone, to 1e-5.
    Covers a ragged last chunk and cell, one cell, one chunk, and a single token."""
    wl = ssd_synth.scaled(W[1], b=1, L=L, H=4, s=s)
    prm, dt, x, Bm, Cm, h0, dy, dhf = _inputs(wl, seed=12)
    ref = _oracle_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf)
    fwd = oracle.scan(x.float().numpy(), Bm.float().numpy(), Cm.float().numpy(), dt.numpy(), prm["A"].numpy(),
                      prm["D"].numpy(), h0.double().numpy(), s=s, H=wl.H, P=wl.P)
    ck = torch.from_numpy(fwd["h_ckpt"]).float()
    got = _gpu_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf, h_ckpt=ck if L >= s else None, s=s if L >= s else 0)
    _compare(got, ref, TOL["f32"], wl)


@pytest.mark.parametrize("wl", [
    ssd_synth.scaled(W[1], b=2, L=777, H=4, G=2, s=256),                 # tensor-core summaries, two groups
    ssd_synth.scaled(W[1], b=1, L=600, H=2, P=32, N=64, Q=64, s=128),    # bf16 off the tensor-core shape
], ids=["bf16-tc-summaries-two-groups", "bf16-cuda-core-summaries"])
def test_bf16_summary_paths(wl):
    """bf16 inputs through both forms of the chunk summaries (tensor cores at P = 64, N = 128 with
    the group of every head; CUDA cores elsewhere), exact checkpoints, to 1e-5."""
    prm, dt, x, Bm, Cm, h0, dy, dhf = _inputs(wl, seed=14)
    ref = _oracle_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf)
    fwd = oracle.scan(x.float().numpy(), Bm.float().numpy(), Cm.float().numpy(), dt.numpy(), prm["A"].numpy(),
                      prm["D"].numpy(), h0.double().numpy(), s=wl.s, H=wl.H, P=wl.P, G=wl.G)
    ck = torch.from_numpy(fwd["h_ckpt"]).float()
    got = _gpu_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf, h_ckpt=ck, s=wl.s)
    _compare(got, ref, TOL["f32"], wl)


def test_bf16_with_gpu_forward_checkpoints():
    """The training pipeline: the tensor-core forward writes the checkpoints, the backward reads them."""
    wl = ssd_synth.scaled(W[1], b=2, L=2048, H=8, s=512)
    prm, dt, x, Bm, Cm, h0, dy, dhf = _inputs(wl, seed=13)
    ref = _oracle_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf)
    d = "cuda"
    _, _, ck = ssd.scan_forward(x.to(d), Bm.to(d), Cm.to(d), dt.to(d), prm["A"].to(d), prm["D"].to(d), h0.to(d),
                                H=wl.H, Q=wl.Q, s=wl.s)
    got = _gpu_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf, h_ckpt=ck.cpu(), s=wl.s)
    _compare(got, ref, TOL["bf16"], wl)


def test_without_checkpoints_groups_and_defaults():
    """No checkpoints (states rebuilt from a zero h0), two groups, no dh_final, a ragged L."""
    wl = ssd_synth.scaled(W[0], b=2, L=700, H=4, G=2, P=32, N=16, Q=32, s=0)
    prm, dt, x, Bm, Cm, _, dy, _ = _inputs(wl, seed=14, h0=False)
    ref = _oracle_bwd(wl, prm, dt, x, Bm, Cm, None, dy, None)
    got = _gpu_bwd(wl, prm, dt, x, Bm, Cm, None, dy, None)
    _compare(got, ref, TOL["f32"], wl)


def test_cells_and_full_agree_on_gpu():
    """The same gradients with and without checkpoints (fp32, P = N = 128)."""
    wl = ssd_synth.scaled(W[0], b=1, L=512, H=2, P=128, N=128, Q=64, s=128)
    prm, dt, x, Bm, Cm, h0, dy, dhf = _inputs(wl, seed=15)
    ref = _oracle_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf)
    fwd = oracle.scan(x.numpy(), Bm.numpy(), Cm.numpy(), dt.numpy(), prm["A"].numpy(), prm["D"].numpy(),
                      h0.double().numpy(), s=wl.s, H=wl.H, P=wl.P)
    a = _gpu_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf, h_ckpt=torch.from_numpy(fwd["h_ckpt"]).float(), s=wl.s)
    b = _gpu_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf)
    _compare(a, ref, TOL["f32"], wl)
    _compare(b, ref, TOL["f32"], wl)
    for k in KEYS:
        assert rel_l2(a[k], b[k]) <= 1e-5, k


def test_03b_shape_all_heads():
    """The 0.3B mixer shape (H = 32, P = 64, N = 128), L = 2048, s = 1024; the oracle recomputes per cell."""
    wl = ssd_synth.scaled(W[1], L=2048)
    prm, dt, x, Bm, Cm, h0, dy, dhf = _inputs(wl, seed=16)
    args = (x.float().numpy(), Bm.float().numpy(), Cm.float().numpy(), dt.numpy(), prm["A"].numpy(),
            prm["D"].numpy())
    fwd = oracle.scan(*args, h0.double().numpy(), s=wl.s, H=wl.H, P=wl.P)
    ref = oracle.scan_backward(*args, dy.float().numpy().reshape(wl.b, wl.L, wl.H, wl.P), h0=h0.double().numpy(),
                               h_ckpt=fwd["h_ckpt"], dh_final=dhf.double().numpy(), s=wl.s, H=wl.H, P=wl.P)
    got = _gpu_bwd(wl, prm, dt, x, Bm, Cm, h0, dy, dhf, h_ckpt=torch.from_numpy(fwd["h_ckpt"]).float(), s=wl.s)
    _compare(got, ref, TOL["f32"], wl)


def test_empty_sequence():
    """L = 0: dh0 = dh_final and zero parameter gradients."""
    wl = ssd_synth.scaled(W[1], b=2, L=0, H=2, s=0)
    d = "cuda"
    x = torch.zeros(2, 0, 128, dtype=torch.bfloat16, device=d)
    Bm = torch.zeros(2, 0, 128, dtype=torch.bfloat16, device=d)
    dt = torch.zeros(2, 0, 2, device=d)
    A = -torch.ones(2, device=d)
    D = torch.ones(2, device=d)
    dy = torch.zeros(2, 0, 128, dtype=torch.bfloat16, device=d)
    dhf = torch.randn(2, 2, 64, 128, device=d)
    out = ssd.scan_backward(x, Bm, Bm, dt, A, D, dy, dh_final=dhf, H=2)
    ssd.sync_status()
    assert torch.equal(out["dh0"], dhf)
    assert torch.all(out["dA"] == 0) and torch.all(out["dD"] == 0)


def test_full_size_bench_configuration():
    """The configuration the backward bench times: b = 1, L = 16384, 32 heads of P = 64, N = 128,
    s = 1024, no h0, dh_final given, the caller's workspace and output buffers (the no-allocation
    form).  Checkpoints come from the oracle's exact forward, so every gradient, dB and dC summed
    over the 32 heads included, is held to 1e-5 against the oracle's reverse mode per cell."""
    wl = ssd_synth.BY_NAME["mamba2-0.3b-L16k"]
    prm, dt, x, Bm, Cm, _, dy, dhf = _inputs(wl, seed=17, h0=False)
    args = (x.float().numpy(), Bm.float().numpy(), Cm.float().numpy(), dt.numpy(), prm["A"].numpy(),
            prm["D"].numpy())
    fwd = oracle.scan(*args, None, s=wl.s, H=wl.H, P=wl.P)
    ref = oracle.scan_backward(*args, dy.float().numpy().reshape(wl.b, wl.L, wl.H, wl.P), h0=None,
                               h_ckpt=fwd["h_ckpt"], dh_final=dhf.double().numpy(), s=wl.s, H=wl.H, P=wl.P)
    d = "cuda"
    ws = torch.empty(ssd.backward_workspace_size(wl.b, wl.L, wl.H, wl.P, wl.N), dtype=torch.uint8, device=d)
    out = {"dx": torch.empty(wl.b, wl.L, wl.H, wl.P, device=d), "dB": torch.empty(wl.b, wl.L, wl.G, wl.N, device=d),
           "dC": torch.empty(wl.b, wl.L, wl.G, wl.N, device=d), "ddt": torch.empty(wl.b, wl.L, wl.H, device=d),
           "dA": torch.empty(wl.H, device=d), "dD": torch.empty(wl.H, device=d),
           "dh0": torch.empty(wl.b, wl.H, wl.P, wl.N, device=d)}
    ck = torch.from_numpy(fwd["h_ckpt"]).float().to(d)
    ssd.scan_backward(x.to(d), Bm.to(d), Cm.to(d), dt.to(d), prm["A"].to(d), prm["D"].to(d), dy.to(d), h_ckpt=ck,
                      dh_final=dhf.to(d), H=wl.H, G=wl.G, s=wl.s, workspace=ws, out=out)
    ssd.sync_status()
    _compare({k: host(v) for k, v in out.items()}, ref, TOL["f32"], wl)
