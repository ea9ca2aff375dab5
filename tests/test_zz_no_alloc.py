"""ssd_scan_forward_static_scratch: the scan for callers that cannot allocate.

Some callers may not call cudaMalloc: code running under a memory pool that
forbids new allocations, or plugin code that is only handed its input and
output buffers.  For them the library offers a variant of ssd_scan_forward
whose scratch is a fixed array compiled into the library.  These tests call
it through the C ABI, twice in a row on different inputs (the array keeps the
previous call's contents), and check each result against the ordinary entry
point with a caller-provided workspace.  Both run the same kernels on the same
inputs with the same stripe plan, so the results must be bitwise equal: any
stale scratch read from the previous call would show.  This file is collected
last on purpose.
"""
import ctypes

import pytest
import torch

import mamba_selective_state_causal_b200 as ssd
import ssd_synth
from parity_util import rel_l2, host

W1 = ssd_synth.WORKLOADS[1]      # 0.3B head shape: P=64, N=128, Q=128, bf16


def _static_scan(x, Bm, Cm, dt, A, D, h0, wl):
    """Call ssd_scan_forward_static_scratch through the C ABI (no workspace)."""
    b, L = x.shape[0], x.shape[1]
    y = torch.empty(b, L, wl.H, wl.P, dtype=x.dtype, device="cuda")
    hf = torch.empty(b, wl.H, wl.P, wl.N, dtype=torch.float32, device="cuda")
    hc = torch.empty(b, L // wl.s, wl.H, wl.P, wl.N, dtype=torch.float32, device="cuda")
    a = ssd.ScanArgs()
    a.dtype = ssd.SSD_BF16; a.b = b; a.L = L; a.H = wl.H; a.P = wl.P; a.N = wl.N; a.G = wl.G
    a.Q = wl.Q; a.s = wl.s
    a.x = x.data_ptr(); a.x_batch_stride = x.stride(0); a.x_row_stride = x.stride(1)
    a.B = Bm.data_ptr(); a.B_batch_stride = Bm.stride(0); a.B_row_stride = Bm.stride(1)
    a.C = Cm.data_ptr(); a.C_batch_stride = Cm.stride(0); a.C_row_stride = Cm.stride(1)
    a.dt = dt.data_ptr(); a.A = A.data_ptr(); a.D = D.data_ptr(); a.h0 = h0.data_ptr()
    y2 = y.view(b, L, wl.H * wl.P)
    a.y = y.data_ptr(); a.y_batch_stride = y2.stride(0); a.y_row_stride = y2.stride(1)
    a.h_final = hf.data_ptr(); a.h_ckpt = hc.data_ptr()
    a.workspace = None; a.workspace_bytes = 0
    rc = ssd.lib().ssd_scan_forward_static_scratch(ctypes.byref(a),
                                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, ssd.lib().ssd_last_error_string()
    return y, hf, hc


@pytest.mark.gpu
def test_static_scratch_scan_matches_workspace_scan_twice():
    wl = ssd_synth.scaled(W1, L=16384)     # needs about 20 MiB of scratch (limit 80 MiB)
    for seed in (11, 12):                  # two calls in a row, different inputs
        prm = ssd_synth.make_params(wl, seed=seed)
        x, Bm, Cm = (t.cuda() for t in ssd_synth.make_xbc(wl, seed=seed))
        dt = ssd_synth.make_dt(wl, prm["dt_bias"], seed=seed).cuda()
        A, D = prm["A"].cuda(), prm["D"].cuda()
        h0 = ssd_synth.make_h0(wl, seed=seed, scale=0.5).cuda()
        ys, hs, cs = _static_scan(x, Bm, Cm, dt, A, D, h0, wl)
        ssd.sync_status()
        yw, hw, cw = ssd.scan_forward(x, Bm, Cm, dt, A, D, h0, H=wl.H, G=wl.G, Q=wl.Q, s=wl.s)
        ssd.sync_status()
        for name, got, ref in (("y", ys, yw), ("h_final", hs, hw), ("h_ckpt", cs, cw)):
            assert torch.equal(got, ref), f"{name}: relL2 {rel_l2(host(got), host(ref))}"


def test_static_scratch_rejects_shapes_beyond_its_size():
    """A shape whose scratch need exceeds the compiled-in array is refused up front."""
    a = ssd.ScanArgs()
    a.dtype = ssd.SSD_BF16; a.b = 2; a.L = 262144; a.H = 64; a.P = 64; a.N = 128; a.G = 1
    a.Q = 128; a.s = 2048
    assert ssd.workspace_size(2, 262144, 64, 64, 128, 128) > 80 << 20
    rc = ssd.lib().ssd_scan_forward_static_scratch(ctypes.byref(a), None)
    assert rc == 9
    assert b"80" in ssd.lib().ssd_last_error_string() or b"bytes" in ssd.lib().ssd_last_error_string()
