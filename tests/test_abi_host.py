"""Host-side checks of the C ABI: the library builds, loads, exports every
symbol include/ssd.h declares, sizes its workspace, and rejects bad arguments
before launching anything.  No call here reaches a GPU kernel."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")


@pytest.fixture(scope="module")
def ssd():
    import __graft_entry__
    __graft_entry__.build()
    import mamba_selective_state_causal_b200 as pkg
    return pkg


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"SSD_API\s+[\w\s\*]+?\b(ssd_\w+)\s*\(", text)


def test_header_declares_entry_points():
    names = declared_symbols()
    for n in ["ssd_conv_forward", "ssd_scan_forward", "ssd_stream_forward",
              "ssd_scan_workspace_size", "ssd_sync_status", "ssd_last_error_string", "ssd_version"]:
        assert n in names


def test_library_exports_every_declared_symbol(ssd):
    out = subprocess.run(["nm", "-D", "--defined-only", ssd.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ssd_\w+)", out))
    missing = [n for n in declared_symbols() if n not in exported]
    assert not missing, missing
    lib = ssd.lib()
    for n in declared_symbols():
        assert hasattr(lib, n)
    assert lib.ssd_version() >= 100


def _plan_bytes(b, L, H, P, N, Q, nsm=148):
    """Workspace of the stripe plan: the stripe length (whole chunks) minimising
    waves x (chunks per stripe + 2), waves = ceil(b * stripes * head pairs / SMs),
    fewest stripes among equals.  Without a GPU the library assumes 148 SMs."""
    if b <= 0 or L <= 0:
        return 0
    nch = -(-L // Q)
    hp = H // 2 if H % 2 == 0 else H
    best = None
    for ns in range(1, min(nch, 16384) + 1):
        tc = -(-nch // ns)
        if -(-nch // tc) != ns:
            continue
        cost = -(-(b * ns * hp) // nsm) * (tc + 2)
        if best is None or cost < best[0]:
            best = (cost, tc)
    ns = -(-L // (best[1] * Q))
    r = lambda v: (v + 255) // 256 * 256
    stripes = 0 if ns <= 1 else 2 * r(4 * b * ns * H * P * N) + r(4 * b * ns * H)
    # followed by room for the effective dt [b][L][H] fp32 (used when dt_bias / softplus / a clamp is asked)
    return r(stripes) + r(4 * b * L * H)


def test_plan_fills_whole_waves():
    """The 0.3B 131072-token segment: 9 stripes x 16 head pairs = 144 CTAs, one wave of 148 SMs."""
    stripes = 2 * 4 * 9 * 32 * 64 * 128 + 9 * 32 * 4 + 256 - (9 * 32 * 4) % 256
    assert _plan_bytes(1, 131072, 32, 64, 128, 128) == stripes + 4 * 131072 * 32


@pytest.mark.parametrize("shape", [(1, 16384, 32, 64, 128, 128), (1, 131072, 32, 64, 128, 128),
                                   (2, 262144, 64, 64, 128, 128), (4, 65536, 80, 64, 128, 128),
                                   (1, 256, 2, 16, 16, 32), (1, 100, 2, 16, 16, 32), (3, 0, 2, 16, 16, 32)])
def test_workspace_size(ssd, shape):
    assert ssd.workspace_size(*shape) == _plan_bytes(*shape)


def _scan_args(ssd, **kw):
    a = ssd.ScanArgs()
    base = dict(dtype=1, b=1, L=256, H=2, P=64, N=128, G=1, Q=128, s=0,
                x=0x10000, x_batch_stride=256 * 384, x_row_stride=384,
                B=0x20000, B_batch_stride=256 * 384, B_row_stride=384,
                C=0x30000, C_batch_stride=256 * 384, C_row_stride=384,
                dt=0x40000, A=0x50000, D=None, h0=None,
                y=0x60000, y_batch_stride=256 * 128, y_row_stride=128,
                h_final=None, h_ckpt=None, workspace=None, workspace_bytes=0)
    base.update(kw)
    for k, v in base.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("change,code", [
    (dict(dtype=7), 5),
    (dict(Q=48), 2),
    (dict(s=100), 2),
    (dict(P=24), 2),
    (dict(N=256), 2),
    (dict(H=3, G=2), 2),
    (dict(b=-1), 2),
    (dict(x=None), 1),
    (dict(dt=None), 1),
    (dict(A=None), 1),
    (dict(y=None), 1),
    (dict(x=0x10002), 3),
    (dict(x_row_stride=385), 3),
    (dict(y_row_stride=64), 4),
    (dict(b=2, x_batch_stride=384), 4),
    (dict(L=1024, H=32, x_row_stride=4096 + 256, y_row_stride=2048 * 2, workspace=None), 9),
])
def test_scan_rejects_bad_arguments(ssd, change, code):
    a = _scan_args(ssd, **change)
    rc = ssd.lib().ssd_scan_forward(ctypes.byref(a), None)
    assert rc == code, (rc, ssd.lib().ssd_last_error_string())
    assert ssd.lib().ssd_last_error_string()


def test_conv_rejects_bad_arguments(ssd):
    L = ssd.lib()
    # C_ch not a multiple of 8 for bf16
    assert L.ssd_conv_forward(0x1000, 120, 12, 0x2000, None, None, None, 0x3000, 120, 12,
                              1, 10, 12, 1, None) == 2
    # misaligned u
    assert L.ssd_conv_forward(0x1008, 160, 16, 0x2000, None, None, None, 0x3000, 160, 16,
                              1, 10, 16, 1, None) == 3
    # missing weights
    assert L.ssd_conv_forward(0x1000, 160, 16, None, None, None, None, 0x3000, 160, 16,
                              1, 10, 16, 1, None) == 1
    # bad dtype
    assert L.ssd_conv_forward(0x1000, 160, 16, 0x2000, None, None, None, 0x3000, 160, 16,
                              1, 10, 16, 9, None) == 5
    # b == 0 is a no-op
    assert L.ssd_conv_forward(None, 0, 0, None, None, None, None, None, 0, 0, 0, 10, 16, 1, None) == 0


def test_stream_without_v_needs_its_workspace(ssd):
    """v = NULL keeps the conv output in the workspace (ssd_stream_workspace_size): the
    scan's workspace, then [b][L][C_ch] of the I/O dtype."""
    a = ssd.StreamArgs()
    a.dtype = 1; a.b = 1; a.L = 64; a.H = 2; a.P = 64; a.N = 128; a.G = 1; a.Q = 128; a.s = 0
    a.u = 0x1000; a.u_row_stride = 384; a.u_batch_stride = 64 * 384
    a.conv_w = 0x2000; a.v = None
    assert ssd.lib().ssd_stream_forward(ctypes.byref(a), None) == 9
    scan = ssd.workspace_size(2, 131072, 32, 64, 128, 128)
    v = 2 * 131072 * (32 * 64 + 256)
    bf = ssd.stream_workspace_size(2, 131072, 32, 64, 128, 1, 128, ssd.SSD_BF16)
    assert scan + 2 * v <= bf < scan + 2 * v + 1024
    f32 = ssd.stream_workspace_size(2, 131072, 32, 64, 128, 1, 128, ssd.SSD_F32)
    assert scan + 4 * v <= f32 < scan + 4 * v + 1024
