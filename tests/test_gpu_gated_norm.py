"""GPU gated RMS norm (ssd_gated_rmsnorm_forward) against the CPU oracle.

bf16 outputs are rounded on both sides; the GPU's fp32 arithmetic may round
an element the other way only where the exact value sits next to a bf16
rounding boundary, so nearly every element must agree bitwise.
"""
import numpy as np
import pytest
import torch

import mamba_selective_state_causal_b200 as ssd
import oracle
import ssd_synth
from parity_util import TOL, host, rel_l2

pytestmark = pytest.mark.gpu


def _gen(shape, dtype, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(dtype)


def _check(got, ref, dtype):
    got = host(got).astype(np.float32)
    if dtype == torch.bfloat16:
        assert rel_l2(got, ref) <= TOL["bf16"]
        assert np.mean(got == ref) >= 0.99, np.mean(got == ref)
    else:
        assert rel_l2(got, ref) <= TOL["f32"]


@pytest.mark.parametrize("dtype,d,group,rows", [
    (torch.bfloat16, 2048, 0, 2000),      # the 0.3B d_inner, one group (a warp per row)
    (torch.bfloat16, 2048, 512, 999),     # four groups of 512, a warp per row
    (torch.bfloat16, 768, 256, 333),      # three chunks of 256, a warp per row
    (torch.bfloat16, 5120, 640, 300),     # the 2.7B d_inner, eight groups
    (torch.float32, 256, 64, 777),
    (torch.float32, 8, 8, 5),
    (torch.bfloat16, 8192, 0, 64),        # the largest row
])
def test_norm_matches_oracle(dtype, d, group, rows):
    y = _gen((rows, d), dtype, 1)
    z = _gen((rows, d), dtype, 2, scale=3.0)
    w = _gen((d,), torch.float32, 3)
    out = ssd.gated_rmsnorm(y.cuda(), z.cuda(), w.cuda(), eps=1e-5, group_size=group)
    ssd.sync_status()
    ref = oracle.gated_rmsnorm(y.float().numpy(), z.float().numpy(), w.numpy(), eps=1e-5,
                               group=group or d, io_round="bf16" if dtype == torch.bfloat16 else "f32")
    _check(out, ref, dtype)


def test_norm_strided_gate_and_in_place():
    """z a column slice of a wider projection; out written over y."""
    b, L, d = 2, 300, 2048
    y = _gen((b, L, d), torch.bfloat16, 4).cuda()
    zx = _gen((b, L, 3 * d), torch.bfloat16, 5).cuda()
    z = zx[:, :, d:2 * d]
    w = _gen((d,), torch.float32, 6).cuda()
    ref = oracle.gated_rmsnorm(host(y), host(z), host(w), eps=1e-6, io_round="bf16")
    out = ssd.gated_rmsnorm(y, z, w, eps=1e-6, out=y)
    ssd.sync_status()
    assert out.data_ptr() == y.data_ptr()
    _check(y, ref, torch.bfloat16)


def test_norm_after_the_scan():
    """The block's tail on the layer output: y from the tensor-core scan, then the gated norm."""
    wl = ssd_synth.scaled(ssd_synth.WORKLOADS[1], L=1000, H=8)
    prm = ssd_synth.make_params(wl)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"])
    x, Bm, Cm = ssd_synth.make_xbc(wl)
    z = _gen((wl.b, wl.L, wl.d_inner), torch.bfloat16, 7)
    w = _gen((wl.d_inner,), torch.float32, 8)
    d = "cuda"
    y, _, _ = ssd.scan_forward(x.to(d), Bm.to(d), Cm.to(d), dt.to(d), prm["A"].to(d), prm["D"].to(d), H=wl.H,
                               Q=wl.Q, s=0)
    out = ssd.gated_rmsnorm(y.reshape(wl.b, wl.L, -1), z.to(d), w.to(d))
    ssd.sync_status()
    ys = oracle.scan(x.float().numpy(), Bm.float().numpy(), Cm.float().numpy(), dt.numpy(), prm["A"].numpy(),
                     prm["D"].numpy(), s=0, H=wl.H, P=wl.P, want_ckpt=False)["y"]
    ref = oracle.gated_rmsnorm(ys.reshape(wl.b, wl.L, -1), z.float().numpy(), w.numpy(), io_round="bf16")
    assert rel_l2(host(out).astype(np.float32), ref) <= TOL["bf16"]


def test_norm_bench_configuration_sampled_rows():
    """The configuration the norm bench times: 131072 rows of 2048 (the 0.3B d_inner), bf16, one
    group, so that each warp of the 296-CTA grid walks about 55 rows; the first and last 64 rows
    and every 61st row between them against the oracle, row by row."""
    rows, d = 131072, 2048
    y = _gen((rows, d), torch.bfloat16, 7)
    z = _gen((rows, d), torch.bfloat16, 8, scale=3.0)
    w = _gen((d,), torch.float32, 9)
    out = torch.empty(rows, d, dtype=torch.bfloat16, device="cuda")
    ssd.gated_rmsnorm(y.cuda(), z.cuda(), w.cuda(), eps=1e-5, out=out)
    ssd.sync_status()
    idx = np.unique(np.r_[0:64, 64:rows - 64:61, rows - 64:rows])
    ref = oracle.gated_rmsnorm(y[idx].float().numpy(), z[idx].float().numpy(), w.numpy(), eps=1e-5,
                               io_round="bf16")
    _check(out[torch.from_numpy(idx).cuda()], ref, torch.bfloat16)
