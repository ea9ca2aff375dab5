"""Host side of ssd_scan_backward: workspace size and argument checks (no GPU needed).

Every rejected call returns before anything touches the device.
"""
import ctypes

import pytest


@pytest.fixture(scope="module")
def ssd():
    import __graft_entry__
    __graft_entry__.build()
    import mamba_selective_state_causal_b200 as pkg
    return pkg


def _round256(v):
    return (v + 255) // 256 * 256


def _bwd_bytes(b, L, H, P, N):
    """Two P x N fp32 states per (64-token chunk, head), three fp32 scalars per
    (chunk, head), two N-vectors of fp32 per (token, head)."""
    if b <= 0 or L <= 0:
        return 0
    nch = -(-L // 64)
    states = 4 * b * H * nch * P * N
    per_chunk = 4 * b * H * nch
    per_token = 4 * b * L * H * N
    return 2 * _round256(states) + 3 * _round256(per_chunk) + 2 * _round256(per_token)


@pytest.mark.parametrize("shape", [(1, 16384, 32, 64, 128), (2, 1000, 4, 16, 32), (1, 1, 1, 16, 16),
                                   (0, 64, 2, 16, 16), (1, 0, 2, 16, 16)])
def test_backward_workspace_size(ssd, shape):
    assert ssd.backward_workspace_size(*shape) == _bwd_bytes(*shape)


def _bwd_args(ssd, **kw):
    a = ssd.ScanBwdArgs()
    base = dict(dtype=1, b=1, L=256, H=2, P=64, N=128, G=1, s=128,
                x=0x10000, x_batch_stride=256 * 384, x_row_stride=384,
                B=0x20000, B_batch_stride=256 * 384, B_row_stride=384,
                C=0x30000, C_batch_stride=256 * 384, C_row_stride=384,
                dt=0x40000, A=0x50000, D=None, h0=None, h_ckpt=0x70000,
                dy=0x60000, dy_batch_stride=256 * 128, dy_row_stride=128, dh_final=None,
                dx=0x80000, dB=0x90000, dC=0xa0000, ddt=0xb0000, dA=0xc0000, dD=None, dh0=None,
                workspace=None, workspace_bytes=0)
    base.update(kw)
    for k, v in base.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("change,code", [
    (dict(dtype=3), 5),
    (dict(s=96), 2),                  # checkpoint stride not a multiple of 64
    (dict(s=0), 2),                   # checkpoints without a stride
    (dict(P=48), 2),
    (dict(H=3, G=2), 2),
    (dict(x=None), 1),
    (dict(dy=None), 1),
    (dict(dx=None), 1),
    (dict(dA=None), 1),
    (dict(dt=None), 1),
    (dict(dy=0x60008), 3),
    (dict(dy_row_stride=100), 4),
    (dict(dh0=0x80004), 3),
    (dict(), 9),                      # no workspace
])
def test_backward_rejects_bad_arguments(ssd, change, code):
    a = _bwd_args(ssd, **change)
    rc = ssd.lib().ssd_scan_backward(ctypes.byref(a), None)
    assert rc == code, (rc, ssd.lib().ssd_last_error_string())
    assert ssd.lib().ssd_last_error_string()


def test_backward_without_checkpoints_ignores_s(ssd):
    """h_ckpt NULL: s is not checked (the states come from h0); the call then only lacks its workspace."""
    a = _bwd_args(ssd, h_ckpt=None, s=96)
    assert ssd.lib().ssd_scan_backward(ctypes.byref(a), None) == 9
