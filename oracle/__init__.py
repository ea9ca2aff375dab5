"""Python access to the CPU oracle (ssd_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only the test-suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The GPU
library never calls it, and it imports nothing from the GPU library.

All arithmetic lives in the C file; this module only marshals numpy arrays
(float32 inputs holding the exact I/O-dtype values, float64 outputs).
"""
import ctypes

import numpy as np

from .build import build as _build

_lib = None


def _bind(path):
    lib = ctypes.CDLL(path)
    f32p = ctypes.POINTER(ctypes.c_float)
    f64p = ctypes.POINTER(ctypes.c_double)
    i32p = ctypes.POINTER(ctypes.c_int)
    i64 = ctypes.c_int64
    lib.oracle_conv.argtypes = [ctypes.c_int, i64, ctypes.c_int, f32p, f32p, f32p,
                                f32p, ctypes.c_int, f32p, f32p]
    lib.oracle_conv.restype = None
    lib.oracle_scan.argtypes = [ctypes.c_int, i64, ctypes.c_int, ctypes.c_int,
                                ctypes.c_int, ctypes.c_int, i64,
                                f32p, i64, i64, f32p, i64, i64, f32p, i64, i64,
                                f32p, f32p, f32p, f64p, i32p, ctypes.c_int,
                                f64p, f64p, f64p]
    lib.oracle_scan.restype = None
    lib.oracle_scan_backward.argtypes = [ctypes.c_int, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, i64,
                                         f32p, i64, i64, f32p, i64, i64, f32p, i64, i64,
                                         f32p, f32p, f32p, f64p, f64p, f64p, f64p,
                                         f64p, f64p, f64p, f64p, f64p, f64p, f64p]
    lib.oracle_scan_backward.restype = None
    lib.oracle_layer_backward.argtypes = [ctypes.c_int, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, i64, f32p, f32p, f32p, f32p, f32p, f32p, f32p,
                                          f64p, f64p, f32p, f64p, f64p, f64p, ctypes.c_int,
                                          f64p, f64p, f64p, f64p, f64p, f64p, f64p, f64p]
    lib.oracle_layer_backward.restype = None
    lib.oracle_gated_rmsnorm.argtypes = [i64, ctypes.c_int, ctypes.c_int, f32p, i64, f32p, i64, f32p,
                                         ctypes.c_double, ctypes.c_int, f32p, i64]
    lib.oracle_gated_rmsnorm.restype = None
    lib.oracle_round_bf16.argtypes = [ctypes.c_double]
    lib.oracle_round_bf16.restype = ctypes.c_double
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(_build())
    return _lib


def use_library(path):
    """Point this module at another build of the oracle source (returns the old one).

    Used by the mutation test, which compiles a deliberately broken copy of
    ssd_oracle.c and checks that the pins reject it.
    """
    global _lib
    old = _lib
    _lib = _bind(path) if isinstance(path, str) else path
    return old


def _f32(a):
    if a is None:
        return None
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a


def _p32(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def _p64(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


IO_ROUND = {"none": 0, "f32": 1, "bf16": 2}


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def round_bf16(values):
    """Round each float64 value to the nearest bfloat16 (ties to even)."""
    lib = _load()
    flat = np.asarray(values, dtype=np.float64).ravel()
    out = np.array([lib.oracle_round_bf16(float(v)) for v in flat])
    return out.reshape(np.shape(values))


def conv(u, w, bias=None, tail_in=None, io_round="none"):
    """Causal depthwise conv1d (kernel 4) + SiLU.

    u: [b, L, Cch]; w: [Cch, 4]; bias: [Cch] or None; tail_in: [b, 3, Cch] or None.
    Returns (v [b, L, Cch] float32 rounded per ``io_round``, tail_out [b, 3, Cch]).
    """
    lib = _load()
    u = _f32(u)
    b, L, cch = u.shape
    w = _f32(w)
    assert w.shape == (cch, 4)
    bias = _f32(bias)
    tail_in = _f32(tail_in)
    if tail_in is not None:
        assert tail_in.shape == (b, 3, cch)
    v = np.empty((b, L, cch), dtype=np.float32)
    tail_out = np.empty((b, 3, cch), dtype=np.float32)
    lib.oracle_conv(b, L, cch, _p32(u), _p32(w), _p32(bias), _p32(tail_in),
                    IO_ROUND[io_round], _p32(v), _p32(tail_out))
    return v, tail_out


def scan(x, B, C, dt, A, D=None, h0=None, s=0, heads=None, H=None, P=None, G=1,
         want_ckpt=True):
    """Literal per-token selective-state recurrence in fp64.

    x: [b, L, >= H*P] (x[:, :, h*P + p] for head h), B and C: [b, L, >= G*N]
    (group g occupies columns g*N .. g*N+N-1), dt: [b, L, H], A: [H], D: [H]
    or None, h0: [b, H, P, N] (float64, any exact state) or None.  ``heads`` selects a subset of heads.
    Returns dict y [b, L, nh, P], h_final [b, nh, P, N], h_ckpt [b, L//s, nh, P, N].
    """
    lib = _load()
    x = np.asarray(x)
    B = np.asarray(B)
    C = np.asarray(C)
    b, L = x.shape[0], x.shape[1]
    dt = _f32(dt)
    H = dt.shape[2] if H is None else H
    assert dt.shape == (b, L, H)
    N = B.shape[2] // G
    if P is None:
        P = x.shape[2] // H
    A = _f32(A)
    D = _f32(D)
    if h0 is not None:
        h0 = np.ascontiguousarray(h0, dtype=np.float64)
        assert h0.shape == (b, H, P, N)

    def strided(a):
        a = _f32(a)
        return a, a.shape[1] * a.shape[2], a.shape[2]

    x, xbs, xrs = strided(x)
    B, Bbs, Brs = strided(B)
    C, Cbs, Crs = strided(C)
    if heads is None:
        hsel = None
        nh = H
    else:
        hsel = np.ascontiguousarray(heads, dtype=np.int32)
        nh = len(hsel)
    y = np.empty((b, L, nh, P), dtype=np.float64)
    h_final = np.empty((b, nh, P, N), dtype=np.float64)
    n_ckpt = L // s if s > 0 else 0
    h_ckpt = np.empty((b, n_ckpt, nh, P, N), dtype=np.float64) if want_ckpt else None
    lib.oracle_scan(b, L, H, P, N, G, int(s), _p32(x), xbs, xrs, _p32(B), Bbs, Brs,
                    _p32(C), Cbs, Crs, _p32(dt), _p32(A), _p32(D), _p64(h0),
                    None if hsel is None else hsel.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                    nh, _p64(y), _p64(h_final), _p64(h_ckpt))
    return {"y": y, "h_final": h_final, "h_ckpt": h_ckpt}


def scan_backward(x, B, C, dt, A, D, dy, h0=None, h_ckpt=None, dh_final=None, s=0, H=None, P=None, G=1):
    """Gradients of the recurrence, fp64, by its literal reverse mode.

    Shapes as in ``scan`` (all heads); dy: [b, L, H, P] and dh_final:
    [b, H, P, N] (or None) are the loss's gradients with respect to y and
    h_final.  With ``h_ckpt`` ([b, L//s, H, P, N], the forward's checkpoints)
    and s > 0, each cell of s tokens is recomputed from its checkpoint;
    without it, the states come from one pass over the whole sequence.
    Returns dict dx [b, L, H, P], dB and dC [b, L, G, N] (summed over the
    heads of each group), ddt [b, L, H], dA and dD [H] (summed over b),
    dh0 [b, H, P, N], and the per-head dB_h, dC_h [b, L, H, N].
    """
    lib = _load()
    x, B, C = np.asarray(x), np.asarray(B), np.asarray(C)
    b, L = x.shape[0], x.shape[1]
    dt = _f32(dt)
    H = dt.shape[2] if H is None else H
    N = B.shape[2] // G
    if P is None:
        P = x.shape[2] // H
    A = _f32(A)
    D = _f32(D)

    def strided(a):
        a = _f32(a)
        return a, a.shape[1] * a.shape[2], a.shape[2]

    def f64(a, shape):
        if a is None:
            return None
        a = np.ascontiguousarray(a, dtype=np.float64)
        assert a.shape == shape, (a.shape, shape)
        return a

    x, xbs, xrs = strided(x)
    B, Bbs, Brs = strided(B)
    C, Cbs, Crs = strided(C)
    h0 = f64(h0, (b, H, P, N))
    n_ckpt = L // s if s > 0 else 0
    h_ckpt = f64(h_ckpt, (b, n_ckpt, H, P, N))
    dy = f64(dy, (b, L, H, P))
    dh_final = f64(dh_final, (b, H, P, N))
    dx = np.empty((b, L, H, P))
    dB_h = np.empty((b, L, H, N))
    dC_h = np.empty((b, L, H, N))
    ddt = np.empty((b, L, H))
    dA_b = np.empty((b, H))
    dD_b = np.empty((b, H))
    dh0 = np.empty((b, H, P, N))
    lib.oracle_scan_backward(b, L, H, P, N, G, int(s), _p32(x), xbs, xrs, _p32(B), Bbs, Brs,
                             _p32(C), Cbs, Crs, _p32(dt), _p32(A), _p32(D), _p64(h0), _p64(h_ckpt),
                             _p64(dy), _p64(dh_final), _p64(dx), _p64(dB_h), _p64(dC_h), _p64(ddt),
                             _p64(dA_b), _p64(dD_b), _p64(dh0))
    grp = (np.arange(H) * G) // H
    dB = np.zeros((b, L, G, N))
    dC = np.zeros((b, L, G, N))
    for h in range(H):
        dB[:, :, grp[h]] += dB_h[:, :, h]
        dC[:, :, grp[h]] += dC_h[:, :, h]
    return {"dx": dx, "dB": dB, "dC": dC, "ddt": ddt, "dA": dA_b.sum(0), "dD": dD_b.sum(0),
            "dh0": dh0, "dB_h": dB_h, "dC_h": dC_h}


def layer_backward(u, w, dt, A, D, dy, bias=None, tail_in=None, h0=None, h_ckpt=None, conv_ckpt=None,
                   dh_final=None, dtail_out=None, H=None, P=None, N=None, G=1, s=0, io_round="none"):
    """Gradients of the whole layer (conv1d + SiLU, then the recurrence), fp64, by its
    literal reverse mode.

    Inputs as for ``layer``; dy [b, L, H, P], dh_final [b, H, P, N] and dtail_out
    [b, 3, Cch] (each optional) are the loss's gradients with respect to y,
    h_final and tail_out.  With ``h_ckpt`` [b, L//s, H, P, N] and ``conv_ckpt``
    [b, L//s, 3, Cch] (the state and the 3 rows of u at every checkpoint) and
    s > 0, each cell of s tokens is rebuilt from its own checkpoint and rows;
    without them, from h0 and tail_in over the whole sequence.
    Returns dict du [b, L, Cch], dtail_in [b, 3, Cch], dw [Cch, 4] and dbias
    [Cch] (summed over b), ddt [b, L, H], dA and dD [H] (summed over b), dh0
    [b, H, P, N].
    """
    lib = _load()
    u = _f32(u)
    b, L, cch = u.shape
    assert cch == H * P + 2 * G * N
    w = _f32(w)
    assert w.shape == (cch, 4)
    bias = _f32(bias)
    tail_in = _f32(tail_in)
    dt = _f32(dt)
    assert dt.shape == (b, L, H)
    A = _f32(A)
    D = _f32(D)

    def f64(a, shape):
        if a is None:
            return None
        a = np.ascontiguousarray(a, dtype=np.float64)
        assert a.shape == shape, (a.shape, shape)
        return a

    n_ckpt = L // s if s > 0 else 0
    h0 = f64(h0, (b, H, P, N))
    h_ckpt = f64(h_ckpt, (b, n_ckpt, H, P, N))
    conv_ckpt = _f32(conv_ckpt)
    if conv_ckpt is not None:
        assert conv_ckpt.shape == (b, n_ckpt, 3, cch)
    dy = f64(dy, (b, L, H, P))
    dh_final = f64(dh_final, (b, H, P, N))
    dtail_out = f64(dtail_out, (b, 3, cch))
    du = np.empty((b, L, cch))
    dtail_in = np.empty((b, 3, cch))
    dw_b = np.empty((b, cch, 4))
    dbias_b = np.empty((b, cch))
    ddt = np.empty((b, L, H))
    dA_b = np.empty((b, H))
    dD_b = np.empty((b, H))
    dh0 = np.empty((b, H, P, N))
    lib.oracle_layer_backward(b, L, H, P, N, G, int(s), _p32(u), _p32(w), _p32(bias), _p32(tail_in),
                              _p32(dt), _p32(A), _p32(D), _p64(h0), _p64(h_ckpt), _p32(conv_ckpt),
                              _p64(dy), _p64(dh_final), _p64(dtail_out), IO_ROUND[io_round],
                              _p64(du), _p64(dtail_in), _p64(dw_b), _p64(dbias_b), _p64(ddt),
                              _p64(dA_b), _p64(dD_b), _p64(dh0))
    return {"du": du, "dtail_in": dtail_in, "dw": dw_b.sum(0), "dbias": dbias_b.sum(0), "ddt": ddt,
            "dA": dA_b.sum(0), "dD": dD_b.sum(0), "dh0": dh0}


def gated_rmsnorm(y, z, w, eps=1e-5, group=None, io_round="none"):
    """out = v / sqrt(mean over the group of v^2 + eps) * w with v = y * silu(z), fp64.

    y, z: [..., d] (the exact I/O values), w: [d]; groups of ``group``
    consecutive channels (default: all d).  Returns float32 rounded per
    ``io_round``, shaped like y.
    """
    lib = _load()
    y = _f32(y)
    z = _f32(z)
    shape = y.shape
    d = shape[-1]
    group = d if group is None else group
    assert z.shape == shape and d % group == 0
    y2 = y.reshape(-1, d)
    z2 = z.reshape(-1, d)
    w = _f32(w)
    out = np.empty_like(y2)
    lib.oracle_gated_rmsnorm(y2.shape[0], d, group, _p32(y2), d, _p32(z2), d, _p32(w), float(eps),
                             IO_ROUND[io_round], _p32(out), d)
    return out.reshape(shape)


def dt_effective(dt, dt_bias=None, softplus=False, dt_min=0.0, dt_max=0.0):
    """The step size from a raw dt, fp64: v = dt + dt_bias[h] (bias optional),
    then softplus(v) = log(1 + e^v) when asked, then clamped to [dt_min, dt_max]
    when dt_max > 0.  These are the Mamba-2 block's dt surroundings, which the
    pages leave out (they give dt itself); dt is [..., H]."""
    v = np.asarray(dt, dtype=np.float64)
    if dt_bias is not None:
        v = v + np.asarray(dt_bias, dtype=np.float64)
    if softplus:
        v = np.logaddexp(0.0, v)
    if dt_max > 0:
        v = np.clip(v, dt_min, dt_max)
    return v


def layer(u, w, dt, A, D=None, bias=None, tail_in=None, h0=None, H=None, P=None, N=None,
          G=1, s=0, io_round="none", heads=None, want_ckpt=True):
    """conv1d+SiLU on the packed x|B|C stream, then the recurrence.

    u: [b, L, H*P + 2*G*N] pre-conv stream, channel order x, then B, then C.
    Returns the scan dict plus ``v`` (the rounded conv output) and ``tail_out``.
    """
    v, tail_out = conv(u, w, bias, tail_in, io_round)
    d_inner = H * P
    x = v[:, :, :d_inner]
    Bm = v[:, :, d_inner:d_inner + G * N]
    Cm = v[:, :, d_inner + G * N:d_inner + 2 * G * N]
    out = scan(x, Bm, Cm, dt, A, D, h0, s, heads=heads, H=H, P=P, G=G, want_ckpt=want_ckpt)
    out["v"] = v
    out["tail_out"] = tail_out
    return out
