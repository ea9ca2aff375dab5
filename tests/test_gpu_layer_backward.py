"""GPU backward pass of the whole layer (ssd_layer_backward) against the CPU oracle.

The page's own test of MA-GC (pith.science verdict record for arXiv
2411.19460, skeptic_critique.concrete_test): one block, d = 64, conv kernel 4,
S = 1024 tokens with checkpoints every s = 128, every parameter gradient of the
recompute-from-checkpoints backward against full-storage backpropagation,
relative error <= 1e-5.  Here: the GPU forward (fp32, d_inner = 128 as two
heads of 64) emits the state checkpoints and the conv buffers; the GPU backward
rebuilds each cell from them; the oracle's full backpropagation (fp64, no
checkpoints) is the reference for du, dtail_in, dconv_w, dconv_bias, ddt, dA,
dD and dh0.  The negative control rebuilds the cells with zero conv buffers
(the state checkpoints alone), which the verdict's skeptic_critique.headline
says is inexact.  Also: a bf16 0.3B-head case through the tensor-core
forward, two groups, L < 3 and L = 0.
"""
import numpy as np
import pytest
import torch

import mamba_selective_state_causal_b200 as ssd
import oracle
import ssd_synth
from parity_util import rel_l2, host

pytestmark = pytest.mark.gpu
W = ssd_synth.WORKLOADS
KEYS = ("du", "dtail_in", "dconv_w", "dconv_bias", "ddt", "dA", "dD", "dh0")
ORACLE_KEY = {"dconv_w": "dw", "dconv_bias": "dbias"}


def _case(wl, seed=0):
    prm = ssd_synth.make_params(wl, seed=seed)
    dto, bias = ssd_synth.make_conv_grads(wl, seed=seed)
    prm["bias"] = bias
    u = ssd_synth.make_u(wl, seed=seed)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"], seed=seed)
    h0 = ssd_synth.make_h0(wl, seed=seed, scale=0.5)
    tail = ssd_synth.make_tail(wl, seed=seed)
    dy, dhf = ssd_synth.make_grads(wl, seed=seed)
    return prm, u, dt, h0, tail, dy, dhf, dto


def _gpu(wl, prm, u, dt, h0, tail, dy, dhf, dto, checkpoints=True, zero_buffers=False):
    d = "cuda"
    g = {k: v.to(d) for k, v in prm.items()}
    fwd = ssd.stream_forward(u.to(d), g["w"], dt.to(d), g["A"], g["D"], H=wl.H, P=wl.P, N=wl.N, G=wl.G,
                             Q=wl.Q, s=wl.s if checkpoints else 0, conv_bias=g["bias"], tail_in=tail.to(d),
                             h0=h0.to(d), conv_ckpt=True if checkpoints else None)
    ck, cb = (fwd["h_ckpt"], fwd["conv_ckpt"]) if checkpoints else (None, None)
    if zero_buffers:
        cb = torch.zeros_like(cb)
    got = ssd.layer_backward(u.to(d), g["w"], dt.to(d), g["A"], g["D"], dy.to(d), H=wl.H, P=wl.P, N=wl.N,
                             G=wl.G, s=wl.s if checkpoints else 0, conv_bias=g["bias"], tail_in=tail.to(d),
                             h0=h0.to(d), h_ckpt=ck, conv_ckpt=cb, dh_final=dhf.to(d), dtail_out=dto.to(d))
    ssd.sync_status()
    return got, fwd


def _oracle(wl, prm, u, dt, h0, tail, dy, dhf, dto):
    return oracle.layer_backward(host(u), prm["w"].numpy(), dt.numpy(), prm["A"].numpy(), prm["D"].numpy(),
                                 host(dy).reshape(wl.b, wl.L, wl.H, wl.P), bias=prm["bias"].numpy(),
                                 tail_in=host(tail), h0=h0.double().numpy(), dh_final=dhf.double().numpy(),
                                 dtail_out=dto.double().numpy(), H=wl.H, P=wl.P, N=wl.N, G=wl.G, s=0,
                                 io_round="bf16" if wl.dtype == "bf16" else "f32")


def _errs(got, ref):
    return {k: rel_l2(host(got[k]), ref[ORACLE_KEY.get(k, k)]) for k in KEYS}


# one block, d = 64 (d_inner = 128: two heads of P = 64), conv kernel 4, S = 1024, s = 128, fp32
PAGE_TEST = ssd_synth.scaled(W[0], L=1024, H=2, P=64, N=64, Q=64, s=128)


def test_page_test_cells_from_checkpoints_match_full_backprop():
    case = _case(PAGE_TEST)
    got, fwd = _gpu(PAGE_TEST, *case)
    assert fwd["conv_ckpt"].shape == (1, 1024 // 128, 3, PAGE_TEST.cch)
    u = case[1]
    for k in range(1024 // 128):
        assert torch.equal(fwd["conv_ckpt"][0, k].cpu(), u[0, (k + 1) * 128 - 3:(k + 1) * 128])
    ref = _oracle(PAGE_TEST, *case)
    errs = _errs(got, ref)
    assert all(e <= 1e-5 for e in errs.values()), errs


def test_without_conv_buffers_the_recompute_is_wrong():
    case = _case(PAGE_TEST)
    good, _ = _gpu(PAGE_TEST, *case)
    bad, _ = _gpu(PAGE_TEST, *case, zero_buffers=True)
    ref = _oracle(PAGE_TEST, *case)
    assert max(_errs(good, ref).values()) <= 1e-5
    e = _errs(bad, ref)
    assert e["dconv_w"] > 1e-3 and e["du"] > 1e-4, e


def test_saturated_conv_activations():
    """u and the conv buffer scaled so that the conv's pre-activations reach past the clamp of the
    sigmoid in the conv's reverse mode (|z| beyond 80 on both sides): both tails of silu' in every
    gradient, to 1e-5."""
    wl = ssd_synth.scaled(PAGE_TEST, L=512)
    prm, u, dt, h0, tail, dy, dhf, dto = _case(wl, seed=9)
    u, tail = u * 60.0, tail * 60.0
    # the pre-activations the layer sees: bias + sum_k w[c, k] u[t - 3 + k, c]
    un, tn, w, b = u[0].double().numpy(), tail[0].double().numpy(), prm["w"].double().numpy(), prm["bias"].double().numpy()
    ext = np.concatenate([tn, un], axis=0)
    z = b + sum(w[:, k] * ext[k:k + wl.L] for k in range(4))
    assert (z > 80).any() and (z < -80).any(), (z.min(), z.max())
    case = (prm, u, dt, h0, tail, dy, dhf, dto)
    got, _ = _gpu(wl, *case)
    errs = _errs(got, _oracle(wl, *case))
    assert all(e <= 1e-5 for e in errs.values()), errs


def test_full_recompute_without_checkpoints():
    wl = ssd_synth.scaled(PAGE_TEST, L=1000)
    case = _case(wl, seed=3)
    got, _ = _gpu(wl, *case, checkpoints=False)
    errs = _errs(got, _oracle(wl, *case))
    assert all(e <= 1e-5 for e in errs.values()), errs


def test_two_groups_ragged_cells():
    wl = ssd_synth.scaled(W[0], L=700, H=4, G=2, P=32, N=32, Q=64, s=128)
    case = _case(wl, seed=5)
    got, _ = _gpu(wl, *case)
    errs = _errs(got, _oracle(wl, *case))
    assert all(e <= 1e-5 for e in errs.values()), errs


def test_bf16_tensor_core_forward_checkpoints():
    """bf16 I/O through the tensor-core forward: the checkpoints carry its own error, so the
    bound is the forward's (1e-2)."""
    wl = ssd_synth.scaled(W[1], L=2048, H=4, s=256)
    case = _case(wl, seed=7)
    got, _ = _gpu(wl, *case)
    errs = _errs(got, _oracle(wl, *case))
    assert all(e <= 1e-2 for e in errs.values()), errs


@pytest.mark.parametrize("L", [1, 2, 3])
def test_shorter_than_the_conv(L):
    wl = ssd_synth.scaled(W[0], L=L, H=2, P=16, N=16, Q=32, s=0)
    case = _case(wl, seed=L)
    got, _ = _gpu(wl, *case, checkpoints=False)
    errs = _errs(got, _oracle(wl, *case))
    assert all(e <= 1e-5 for e in errs.values()), errs


def test_empty_sequence():
    wl = ssd_synth.scaled(W[0], L=0, H=2, P=16, N=16, Q=32, s=0)
    prm, u, dt, h0, tail, dy, dhf, dto = _case(wl)
    d = "cuda"
    g = {k: v.to(d) for k, v in prm.items()}
    got = ssd.layer_backward(u.to(d), g["w"], dt.to(d), g["A"], g["D"], dy.to(d), H=wl.H, P=wl.P, N=wl.N,
                             conv_bias=g["bias"], tail_in=tail.to(d), h0=h0.to(d), dh_final=dhf.to(d),
                             dtail_out=dto.to(d))
    ssd.sync_status()
    assert torch.equal(got["dtail_in"].cpu(), dto)
    assert torch.equal(got["dh0"].cpu(), dhf)
    assert float(got["dconv_w"].abs().max()) == 0.0 and float(got["dA"].abs().max()) == 0.0



@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_full_size_bench_configuration(io):
    """The configuration the layer-backward bench times: b = 1, L = 16384, the 0.3B mixer (32 heads
    of P = 64, N = 128, 2304 conv channels), s = 1024, no h0 or tail_in, the caller's workspace,
    then its output buffers (the no-allocation form); bf16 I/O as the bench runs it, and fp32.
    The state checkpoints come from the oracle's exact forward and the conv buffers are the 3 rows
    of u before each cell.  A second call, into the first call's outputs, must reproduce it bit
    for bit (every reduction runs in a fixed order).

    fp32 I/O: every gradient to 1e-5.  bf16 I/O rounds the conv output v to bf16, a decision
    that the GPU takes on an fp32 value and the oracle on an fp64 one, so a few elements of v
    round to the other neighbour (the two are then one bf16 spacing apart, 2^-7 relative at
    most).  The test checks that every element of the GPU's v is a valid rounding (within one
    spacing of the exact SiLU, plus the fp32 rounding of the four-tap sum, plus the hardware
    tanh's approximation of sigma, 2^-12 absolute), that at most 1e-3 of them round the other
    way, and hence that v's relL2 against the oracle's rounding is at most
    sqrt(1e-3) * 2^-7 = 2.5e-4; the gradients, which carry that difference of v with a gain
    of about 2, are held to 5e-4."""
    wl = ssd_synth.scaled(ssd_synth.BY_NAME["mamba2-0.3b-L16k"], dtype=io)
    seed = 18
    prm = ssd_synth.make_params(wl, seed=seed)
    dto, _ = ssd_synth.make_conv_grads(wl, seed=seed)
    u = ssd_synth.make_u(wl, seed=seed)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"], seed=seed)
    dy, dhf = ssd_synth.make_grads(wl, seed=seed)
    un = host(u)
    fwd = oracle.layer(un, prm["w"].numpy(), dt.numpy(), prm["A"].numpy(), prm["D"].numpy(), bias=prm["bias"].numpy(),
                       H=wl.H, P=wl.P, N=wl.N, G=wl.G, s=wl.s, io_round=io)
    cc = torch.stack([u[:, (j + 1) * wl.s - 3:(j + 1) * wl.s] for j in range(wl.L // wl.s)], dim=1)
    ref = oracle.layer_backward(un, prm["w"].numpy(), dt.numpy(), prm["A"].numpy(), prm["D"].numpy(),
                                host(dy).reshape(wl.b, wl.L, wl.H, wl.P), bias=prm["bias"].numpy(),
                                h_ckpt=fwd["h_ckpt"], conv_ckpt=host(cc), dh_final=dhf.double().numpy(),
                                dtail_out=dto.double().numpy(), H=wl.H, P=wl.P, N=wl.N, G=wl.G, s=wl.s,
                                io_round=io)
    d = "cuda"
    g = {k: v.to(d) for k, v in prm.items()}
    gf = ssd.stream_forward(u.to(d), g["w"], dt.to(d), g["A"], g["D"], H=wl.H, P=wl.P, N=wl.N, G=wl.G, Q=wl.Q,
                            s=wl.s, conv_bias=g["bias"])
    ssd.sync_status()
    vg = host(gf["v"]).astype(np.float64)
    vo = np.asarray(fwd["v"], dtype=np.float64)
    if io == "bf16":
        ve = oracle.conv(un, prm["w"].numpy(), prm["bias"].numpy())[0].astype(np.float64)
        # size of the conv's pre-activation terms, for the fp32 rounding of their sum
        w, b = prm["w"].double().numpy(), prm["bias"].double().numpy()
        ext = np.concatenate([np.zeros((wl.b, 3, wl.cch)), un.astype(np.float64)], axis=1)
        zabs = np.abs(b) + sum(np.abs(w[:, k] * ext[:, k:k + wl.L]) for k in range(4))
        z = b + sum(w[:, k] * ext[:, k:k + wl.L] for k in range(4))
        mant, ex = np.frexp(np.abs(ve))
        spacing = np.where(ve == 0.0, 0.0, np.ldexp(1.0, ex - 8))
        bound = spacing + 1.1 * 5 * 2.0 ** -24 * zabs + np.abs(z) * 2.0 ** -12
        over = np.abs(vg - ve) > bound
        assert not over.any(), (int(over.sum()), float(np.abs(vg - ve)[over].max()))
        flips = float(np.mean(vg != vo))
        assert flips <= 1e-3, flips
        ev = rel_l2(vg, vo)
        assert ev <= 2.5e-4, ev
        tol = 5e-4
    else:
        assert rel_l2(vg, vo) <= 1e-6
        tol = 1e-5
    ws = torch.empty(ssd.layer_backward_workspace_size(wl.b, wl.L, wl.H, wl.P, wl.N, wl.G,
                                                      ssd.SSD_BF16 if io == "bf16" else ssd.SSD_F32),
                     dtype=torch.uint8, device=d)
    kw = dict(H=wl.H, P=wl.P, N=wl.N, G=wl.G, s=wl.s, conv_bias=g["bias"],
              h_ckpt=torch.from_numpy(fwd["h_ckpt"]).float().to(d), conv_ckpt=cc.to(d), dh_final=dhf.to(d),
              dtail_out=dto.to(d), workspace=ws)
    args = (u.to(d), g["w"], dt.to(d), g["A"], g["D"], dy.to(d))
    first = ssd.layer_backward(*args, **kw)
    ssd.sync_status()
    snap = {k: host(first[k]).copy() for k in KEYS}
    for v in first.values():
        if torch.is_tensor(v):
            v.fill_(float("nan"))
    again = ssd.layer_backward(*args, out=first, **kw)
    ssd.sync_status()
    errs = _errs(again, ref)
    assert all(e <= tol for e in errs.values()), errs
    for k in KEYS:
        assert np.array_equal(host(again[k]), snap[k]), k
