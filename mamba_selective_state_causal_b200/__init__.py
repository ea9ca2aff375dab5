"""Python binding of the B200 SSD layer library (libssd.so, C ABI in include/ssd.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  torch tensors supply device memory and the CUDA stream.  If the
compiled library is missing, importing the binding's functions raises: there
is no fallback implementation.
"""
import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libssd.so")

SSD_F32, SSD_BF16 = 0, 1
STATUS = {0: "SSD_OK", 1: "SSD_ERR_NULL", 2: "SSD_ERR_SHAPE", 3: "SSD_ERR_ALIGN",
          4: "SSD_ERR_STRIDE", 5: "SSD_ERR_DTYPE", 6: "SSD_ERR_UNSUPPORTED",
          7: "SSD_ERR_LAUNCH", 8: "SSD_ERR_TIMEOUT", 9: "SSD_ERR_WORKSPACE"}

_i64 = ctypes.c_int64
_vp = ctypes.c_void_p


class SSDError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", _i64), ("total_ms", ctypes.c_double)]


class ScanArgs(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("b", ctypes.c_int), ("L", _i64),
                ("H", ctypes.c_int), ("P", ctypes.c_int), ("N", ctypes.c_int),
                ("G", ctypes.c_int), ("Q", ctypes.c_int), ("s", _i64),
                ("x", _vp), ("x_batch_stride", _i64), ("x_row_stride", _i64),
                ("B", _vp), ("B_batch_stride", _i64), ("B_row_stride", _i64),
                ("C", _vp), ("C_batch_stride", _i64), ("C_row_stride", _i64),
                ("dt", _vp), ("A", _vp), ("D", _vp), ("h0", _vp),
                ("y", _vp), ("y_batch_stride", _i64), ("y_row_stride", _i64),
                ("h_final", _vp), ("h_ckpt", _vp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
                ("dt_bias", _vp), ("dt_softplus", ctypes.c_int),
                ("dt_min", ctypes.c_float), ("dt_max", ctypes.c_float)]


class StreamArgs(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("b", ctypes.c_int), ("L", _i64),
                ("H", ctypes.c_int), ("P", ctypes.c_int), ("N", ctypes.c_int),
                ("G", ctypes.c_int), ("Q", ctypes.c_int), ("s", _i64),
                ("u", _vp), ("u_batch_stride", _i64), ("u_row_stride", _i64),
                ("conv_w", _vp), ("conv_bias", _vp), ("tail_in", _vp), ("tail_out", _vp),
                ("v", _vp), ("v_batch_stride", _i64), ("v_row_stride", _i64),
                ("dt", _vp), ("A", _vp), ("D", _vp), ("h0", _vp),
                ("y", _vp), ("y_batch_stride", _i64), ("y_row_stride", _i64),
                ("h_final", _vp), ("h_ckpt", _vp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
                ("dt_bias", _vp), ("dt_softplus", ctypes.c_int),
                ("dt_min", ctypes.c_float), ("dt_max", ctypes.c_float),
                ("conv_ckpt", _vp)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("b", ctypes.c_int),
                ("H", ctypes.c_int), ("P", ctypes.c_int), ("N", ctypes.c_int), ("G", ctypes.c_int),
                ("u", _vp), ("u_batch_stride", _i64),
                ("conv_w", _vp), ("conv_bias", _vp), ("tail_in", _vp), ("tail_out", _vp),
                ("dt", _vp), ("A", _vp), ("D", _vp), ("h_in", _vp), ("h_out", _vp),
                ("y", _vp), ("y_batch_stride", _i64),
                ("dt_bias", _vp), ("dt_softplus", ctypes.c_int),
                ("dt_min", ctypes.c_float), ("dt_max", ctypes.c_float)]


class ScanBwdArgs(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("b", ctypes.c_int), ("L", _i64),
                ("H", ctypes.c_int), ("P", ctypes.c_int), ("N", ctypes.c_int),
                ("G", ctypes.c_int), ("s", _i64),
                ("x", _vp), ("x_batch_stride", _i64), ("x_row_stride", _i64),
                ("B", _vp), ("B_batch_stride", _i64), ("B_row_stride", _i64),
                ("C", _vp), ("C_batch_stride", _i64), ("C_row_stride", _i64),
                ("dt", _vp), ("A", _vp), ("D", _vp), ("h0", _vp), ("h_ckpt", _vp),
                ("dy", _vp), ("dy_batch_stride", _i64), ("dy_row_stride", _i64),
                ("dh_final", _vp),
                ("dx", _vp), ("dB", _vp), ("dC", _vp), ("ddt", _vp), ("dA", _vp), ("dD", _vp),
                ("dh0", _vp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


class LayerBwdArgs(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("b", ctypes.c_int), ("L", _i64),
                ("H", ctypes.c_int), ("P", ctypes.c_int), ("N", ctypes.c_int),
                ("G", ctypes.c_int), ("s", _i64),
                ("u", _vp), ("u_batch_stride", _i64), ("u_row_stride", _i64),
                ("conv_w", _vp), ("conv_bias", _vp), ("tail_in", _vp), ("conv_ckpt", _vp),
                ("dt", _vp), ("A", _vp), ("D", _vp), ("h0", _vp), ("h_ckpt", _vp),
                ("dy", _vp), ("dy_batch_stride", _i64), ("dy_row_stride", _i64),
                ("dh_final", _vp), ("dtail_out", _vp),
                ("du", _vp), ("dtail_in", _vp), ("dconv_w", _vp), ("dconv_bias", _vp),
                ("ddt", _vp), ("dA", _vp), ("dD", _vp), ("dh0", _vp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


_lib = None


def lib():
    """The loaded libssd.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(LIB_PATH)
        L.ssd_conv_forward.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _i64, _i64,
                                       ctypes.c_int, _i64, ctypes.c_int, ctypes.c_int, _vp]
        L.ssd_conv_forward.restype = ctypes.c_int
        L.ssd_scan_forward.argtypes = [ctypes.POINTER(ScanArgs), _vp]
        L.ssd_scan_forward.restype = ctypes.c_int
        L.ssd_stream_forward.argtypes = [ctypes.POINTER(StreamArgs), _vp]
        L.ssd_stream_forward.restype = ctypes.c_int
        L.ssd_decode_step.argtypes = [ctypes.POINTER(DecodeArgs), _vp]
        L.ssd_decode_step.restype = ctypes.c_int
        L.ssd_gated_rmsnorm_forward.argtypes = [_vp, _i64, _vp, _i64, _vp, ctypes.c_float, ctypes.c_int, _vp, _i64,
                                                _i64, ctypes.c_int, ctypes.c_int, _vp]
        L.ssd_gated_rmsnorm_forward.restype = ctypes.c_int
        L.ssd_scan_backward.argtypes = [ctypes.POINTER(ScanBwdArgs), _vp]
        L.ssd_scan_backward.restype = ctypes.c_int
        L.ssd_scan_backward_workspace_size.argtypes = [ctypes.c_int, _i64, ctypes.c_int, ctypes.c_int,
                                                       ctypes.c_int]
        L.ssd_scan_backward_workspace_size.restype = ctypes.c_size_t
        L.ssd_layer_backward.argtypes = [ctypes.POINTER(LayerBwdArgs), _vp]
        L.ssd_layer_backward.restype = ctypes.c_int
        L.ssd_layer_backward_workspace_size.argtypes = [ctypes.c_int, _i64, ctypes.c_int, ctypes.c_int,
                                                        ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.ssd_layer_backward_workspace_size.restype = ctypes.c_size_t
        L.ssd_stream_workspace_size.argtypes = [ctypes.c_int, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.ssd_stream_workspace_size.restype = ctypes.c_size_t
        L.ssd_scan_workspace_size.argtypes = [ctypes.c_int, _i64, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int]
        L.ssd_scan_workspace_size.restype = ctypes.c_size_t
        L.ssd_sync_status.argtypes = [_vp]
        L.ssd_sync_status.restype = ctypes.c_int
        L.ssd_last_error_string.argtypes = []
        L.ssd_last_error_string.restype = ctypes.c_char_p
        L.ssd_version.argtypes = []
        L.ssd_version.restype = ctypes.c_int
        L.ssd_scan_forward_static_scratch.argtypes = [ctypes.POINTER(ScanArgs), _vp]
        L.ssd_scan_forward_static_scratch.restype = ctypes.c_int
        L.ssd_profile_begin.argtypes = []
        L.ssd_profile_begin.restype = ctypes.c_int
        L.ssd_profile_end.argtypes = [ctypes.POINTER(KernelStat), ctypes.c_int,
                                      ctypes.POINTER(ctypes.c_int)]
        L.ssd_profile_end.restype = ctypes.c_int
        _lib = L
    return _lib


def _check(rc):
    if rc != 0:
        raise SSDError(rc, lib().ssd_last_error_string().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return SSD_BF16
    if t.dtype == torch.float32:
        return SSD_F32
    raise TypeError(f"unsupported I/O dtype {t.dtype}")


def _cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")


def _f32(t, name):
    if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()):
        raise TypeError(f"{name} must be a contiguous float32 tensor")
    return t


def workspace_size(b, L, H, P, N, Q):
    return int(lib().ssd_scan_workspace_size(b, L, H, P, N, Q))


def stream_workspace_size(b, L, H, P, N, G, Q, dtype):
    """Workspace bytes of stream_forward without the conv output (keep_v=False)."""
    return int(lib().ssd_stream_workspace_size(b, L, H, P, N, G, Q, dtype))


def alloc_workspace(b, L, H, P, N, Q, device=None):
    n = workspace_size(b, L, H, P, N, Q)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device or "cuda")


def profile_begin():
    """Start timing every kernel the library launches from this thread."""
    _check(lib().ssd_profile_begin())


def profile_end():
    """Stop timing; returns {kernel name: {"launches": n, "total_ms": t}}."""
    cap = 32
    arr = (KernelStat * cap)()
    n = ctypes.c_int(0)
    _check(lib().ssd_profile_end(arr, cap, ctypes.byref(n)))
    return {arr[i].name.decode(): {"launches": int(arr[i].launches), "total_ms": float(arr[i].total_ms)}
            for i in range(min(n.value, cap))}


def sync_status(stream=None):
    _check(lib().ssd_sync_status(_stream(stream)))


def conv_forward(u, w, bias=None, tail_in=None, tail_out=None, v=None, stream=None):
    """v = silu(causal_conv1d_k4(u)); returns (v, tail_out)."""
    _cuda(u, w, bias, tail_in, tail_out, v)
    b, L, cch = u.shape
    if v is None:
        v = torch.empty_like(u)
    _f32(w, "w")
    _f32(bias, "bias")
    rc = lib().ssd_conv_forward(_ptr(u), u.stride(0), u.stride(1), _ptr(w), _ptr(bias),
                                _ptr(tail_in), _ptr(tail_out), _ptr(v), v.stride(0), v.stride(1),
                                b, L, cch, _dtype_code(u), _stream(stream))
    _check(rc)
    return v, tail_out



def _set_dt(a, dt_bias, dt_softplus, dt_limit):
    """The optional dt_bias [H] float32 / softplus / (lo, hi) clamp of the arguments."""
    _cuda(dt_bias)
    _f32(dt_bias, "dt_bias")
    a.dt_bias = dt_bias.data_ptr() if dt_bias is not None else None
    a.dt_softplus = 1 if dt_softplus else 0
    lo, hi = dt_limit if dt_limit is not None else (0.0, 0.0)
    a.dt_min, a.dt_max = float(lo), float(hi)

def scan_forward(x, B, C, dt, A, D=None, h0=None, *, H, G=1, Q=128, s=0, y=None,
                 h_final=None, h_ckpt=None, workspace=None, stream=None, dt_bias=None,
                 dt_softplus=False, dt_limit=None):
    """Chunked selective scan; returns (y, h_final, h_ckpt).

    x: [b, L, >=H*P] view (may be a column slice of the conv output),
    B, C: [b, L, >=G*N] views, dt: [b, L, H] float32, A/D: [H] float32,
    h0: [b, H, P, N] float32 or None.  dt_bias [H] / dt_softplus / dt_limit (lo, hi):
    the kernels use clamp(softplus(dt + dt_bias)) instead of dt (each part optional).
    """
    _cuda(x, B, C, dt, A, D, h0, y, h_final, h_ckpt, workspace)
    b, L = x.shape[0], x.shape[1]
    P = x.shape[2] // H
    N = B.shape[2] // G
    dev = x.device
    if y is None:
        y = torch.empty(b, L, H, P, dtype=x.dtype, device=dev)
    if h_final is None:
        h_final = torch.empty(b, H, P, N, dtype=torch.float32, device=dev)
    if h_ckpt is None and s > 0:
        h_ckpt = torch.empty(b, L // s, H, P, N, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(b, L, H, P, N, Q, dev)
    for t, n in ((dt, "dt"), (A, "A"), (D, "D"), (h0, "h0"), (h_final, "h_final"), (h_ckpt, "h_ckpt")):
        _f32(t, n)
    a = ScanArgs()
    a.dtype = _dtype_code(x); a.b = b; a.L = L; a.H = H; a.P = P; a.N = N; a.G = G; a.Q = Q; a.s = s
    a.x = x.data_ptr(); a.x_batch_stride = x.stride(0); a.x_row_stride = x.stride(1)
    a.B = B.data_ptr(); a.B_batch_stride = B.stride(0); a.B_row_stride = B.stride(1)
    a.C = C.data_ptr(); a.C_batch_stride = C.stride(0); a.C_row_stride = C.stride(1)
    a.dt = dt.data_ptr(); a.A = A.data_ptr(); a.D = D.data_ptr() if D is not None else None
    a.h0 = h0.data_ptr() if h0 is not None else None
    y2 = y.view(b, L, H * P)
    a.y = y.data_ptr(); a.y_batch_stride = y2.stride(0); a.y_row_stride = y2.stride(1)
    a.h_final = h_final.data_ptr() if h_final is not None else None
    a.h_ckpt = h_ckpt.data_ptr() if h_ckpt is not None else None
    a.workspace = workspace.data_ptr(); a.workspace_bytes = workspace.numel() * workspace.element_size()
    _set_dt(a, dt_bias, dt_softplus, dt_limit)
    _check(lib().ssd_scan_forward(ctypes.byref(a), _stream(stream)))
    return y, h_final, h_ckpt


def stream_forward(u, conv_w, dt, A, D=None, *, H, P, N, G=1, Q=128, s=0, conv_bias=None,
                   tail_in=None, tail_out=None, h0=None, v=None, y=None, h_final=None,
                   h_ckpt=None, workspace=None, stream=None, dt_bias=None, dt_softplus=False,
                   dt_limit=None, conv_ckpt=None, keep_v=True):
    """One streamed segment: conv (tail_in -> tail_out), then scan (h0 -> h_final).

    conv_ckpt: a [b, L//s, 3, C_ch] tensor (I/O dtype) to receive the conv buffer at
    every checkpoint, True to allocate one, or None.  keep_v=False (and v None):
    the conv output is not returned, and on the tensor-core shapes the conv of x is
    fused into the scan kernels (the workspace is then ssd_stream_workspace_size)."""
    _cuda(u, conv_w, dt, A, D, conv_bias, tail_in, tail_out, h0, v, y, h_final, h_ckpt, workspace)
    b, L, cch = u.shape
    assert cch == H * P + 2 * G * N, "u must hold x|B|C channels"
    dev = u.device
    if v is None and keep_v:
        v = torch.empty_like(u)
    if y is None:
        y = torch.empty(b, L, H, P, dtype=u.dtype, device=dev)
    if h_final is None:
        h_final = torch.empty(b, H, P, N, dtype=torch.float32, device=dev)
    if tail_out is None:
        tail_out = torch.empty(b, 3, cch, dtype=u.dtype, device=dev)
    if h_ckpt is None and s > 0:
        h_ckpt = torch.empty(b, L // s, H, P, N, dtype=torch.float32, device=dev)
    if workspace is None:
        if v is None:
            n = stream_workspace_size(b, L, H, P, N, G, Q, _dtype_code(u))
            workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=dev)
        else:
            workspace = alloc_workspace(b, L, H, P, N, Q, dev)
    if conv_ckpt is True:
        conv_ckpt = torch.empty(b, L // s if s > 0 else 0, 3, cch, dtype=u.dtype, device=dev)
    a = StreamArgs()
    a.dtype = _dtype_code(u); a.b = b; a.L = L; a.H = H; a.P = P; a.N = N; a.G = G; a.Q = Q; a.s = s
    a.u = u.data_ptr(); a.u_batch_stride = u.stride(0); a.u_row_stride = u.stride(1)
    a.conv_w = conv_w.data_ptr(); a.conv_bias = conv_bias.data_ptr() if conv_bias is not None else None
    a.tail_in = tail_in.data_ptr() if tail_in is not None else None
    a.tail_out = tail_out.data_ptr()
    if v is not None:
        a.v = v.data_ptr(); a.v_batch_stride = v.stride(0); a.v_row_stride = v.stride(1)
    a.dt = dt.data_ptr(); a.A = A.data_ptr(); a.D = D.data_ptr() if D is not None else None
    a.h0 = h0.data_ptr() if h0 is not None else None
    y2 = y.view(b, L, H * P)
    a.y = y.data_ptr(); a.y_batch_stride = y2.stride(0); a.y_row_stride = y2.stride(1)
    a.h_final = h_final.data_ptr()
    a.h_ckpt = h_ckpt.data_ptr() if h_ckpt is not None else None
    a.workspace = workspace.data_ptr(); a.workspace_bytes = workspace.numel()
    _set_dt(a, dt_bias, dt_softplus, dt_limit)
    a.conv_ckpt = conv_ckpt.data_ptr() if conv_ckpt is not None else None
    _check(lib().ssd_stream_forward(ctypes.byref(a), _stream(stream)))
    return {"v": v, "y": y, "h_final": h_final, "h_ckpt": h_ckpt, "tail_out": tail_out, "conv_ckpt": conv_ckpt}


def decode_step(u, conv_w, dt, A, D=None, *, H, P, N, G=1, conv_bias=None, tail_in=None,
                tail_out=None, h_in=None, h_out=None, y=None, stream=None, dt_bias=None,
                dt_softplus=False, dt_limit=None):
    """One token of b streams: u [b, C_ch] (pre-conv x|B|C), dt [b, H].  Returns
    {"y": [b, H, P], "h_out": [b, H, P, N], "tail_out": [b, 3, C_ch]}; h_out may be h_in
    and tail_out may be tail_in (updated in place)."""
    _cuda(u, conv_w, dt, A, D, conv_bias, tail_in, tail_out, h_in, h_out, y)
    b, cch = u.shape
    assert cch == H * P + 2 * G * N, "u must hold x|B|C channels"
    dev = u.device
    if y is None:
        y = torch.empty(b, H, P, dtype=u.dtype, device=dev)
    if h_out is None:
        h_out = torch.empty(b, H, P, N, dtype=torch.float32, device=dev)
    if tail_out is None:
        tail_out = torch.empty(b, 3, cch, dtype=u.dtype, device=dev)
    a = DecodeArgs()
    a.dtype = _dtype_code(u); a.b = b; a.H = H; a.P = P; a.N = N; a.G = G
    a.u = u.data_ptr(); a.u_batch_stride = u.stride(0)
    a.conv_w = conv_w.data_ptr(); a.conv_bias = conv_bias.data_ptr() if conv_bias is not None else None
    a.tail_in = tail_in.data_ptr() if tail_in is not None else None
    a.tail_out = tail_out.data_ptr()
    a.dt = dt.data_ptr(); a.A = A.data_ptr(); a.D = D.data_ptr() if D is not None else None
    a.h_in = h_in.data_ptr() if h_in is not None else None
    a.h_out = h_out.data_ptr()
    a.y = y.data_ptr(); a.y_batch_stride = y.view(b, H * P).stride(0)
    _set_dt(a, dt_bias, dt_softplus, dt_limit)
    _check(lib().ssd_decode_step(ctypes.byref(a), _stream(stream)))
    return {"y": y, "h_out": h_out, "tail_out": tail_out}


def backward_workspace_size(b, L, H, P, N):
    return int(lib().ssd_scan_backward_workspace_size(b, L, H, P, N))


def scan_backward(x, B, C, dt, A, D, dy, h0=None, h_ckpt=None, dh_final=None, *, H, G=1, s=0,
                  workspace=None, out=None, stream=None):
    """Gradients through scan_forward: returns dict dx, dB, dC, ddt, dA, dD, dh0 (float32).

    x, B, C, dt, A, D, h0: the forward's inputs (views as for scan_forward);
    dy: [b, L, >=H*P] (I/O dtype) = dLoss/dy, dh_final: [b, H, P, N] float32
    or None.  h_ckpt: the forward's checkpoints [b, L//s, H, P, N] with stride
    s, or None to rebuild the states from h0 over the whole sequence.
    ``out`` may hold preallocated outputs under the same keys.
    """
    _cuda(x, B, C, dt, A, D, dy, h0, h_ckpt, dh_final, workspace)
    b, L = x.shape[0], x.shape[1]
    P = x.shape[2] // H
    N = B.shape[2] // G
    dev = x.device
    o = dict(out or {})
    shapes = {"dx": (b, L, H, P), "dB": (b, L, G, N), "dC": (b, L, G, N), "ddt": (b, L, H),
              "dA": (H,), "dD": (H,), "dh0": (b, H, P, N)}
    for k, shp in shapes.items():
        if k not in o:
            o[k] = torch.empty(shp, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(backward_workspace_size(b, L, H, P, N), 1), dtype=torch.uint8, device=dev)
    for t, n in ((dt, "dt"), (A, "A"), (D, "D"), (h0, "h0"), (h_ckpt, "h_ckpt"), (dh_final, "dh_final"),
                 *((o[k], k) for k in shapes)):
        _f32(t, n)
    a = ScanBwdArgs()
    a.dtype = _dtype_code(x); a.b = b; a.L = L; a.H = H; a.P = P; a.N = N; a.G = G
    a.s = s if h_ckpt is not None else 0
    a.x = x.data_ptr(); a.x_batch_stride = x.stride(0); a.x_row_stride = x.stride(1)
    a.B = B.data_ptr(); a.B_batch_stride = B.stride(0); a.B_row_stride = B.stride(1)
    a.C = C.data_ptr(); a.C_batch_stride = C.stride(0); a.C_row_stride = C.stride(1)
    a.dt = dt.data_ptr(); a.A = A.data_ptr(); a.D = D.data_ptr() if D is not None else None
    a.h0 = h0.data_ptr() if h0 is not None else None
    a.h_ckpt = h_ckpt.data_ptr() if h_ckpt is not None else None
    dy3 = dy.reshape(b, L, -1) if dy.dim() == 4 else dy
    a.dy = dy3.data_ptr(); a.dy_batch_stride = dy3.stride(0); a.dy_row_stride = dy3.stride(1)
    a.dh_final = dh_final.data_ptr() if dh_final is not None else None
    a.dx = o["dx"].data_ptr(); a.dB = o["dB"].data_ptr(); a.dC = o["dC"].data_ptr()
    a.ddt = o["ddt"].data_ptr(); a.dA = o["dA"].data_ptr()
    a.dD = o["dD"].data_ptr() if o["dD"] is not None else None
    a.dh0 = o["dh0"].data_ptr() if o["dh0"] is not None else None
    a.workspace = workspace.data_ptr(); a.workspace_bytes = workspace.numel()
    _check(lib().ssd_scan_backward(ctypes.byref(a), _stream(stream)))
    return o


def layer_backward_workspace_size(b, L, H, P, N, G=1, dtype=SSD_BF16):
    return int(lib().ssd_layer_backward_workspace_size(b, L, H, P, N, G, dtype))


def layer_backward(u, conv_w, dt, A, D, dy, *, H, P, N, G=1, s=0, conv_bias=None, tail_in=None, h0=None,
                   h_ckpt=None, conv_ckpt=None, dh_final=None, dtail_out=None, workspace=None, out=None,
                   stream=None):
    """Gradients through the whole layer (conv1d + SiLU, then the scan): returns dict du,
    dtail_in, dconv_w, dconv_bias, ddt, dA, dD, dh0 (float32).

    u, conv_w, conv_bias, tail_in, dt, A, D, h0: the forward's inputs (as for
    stream_forward); dy: [b, L, >=H*P] (I/O dtype); dh_final [b, H, P, N] and
    dtail_out [b, 3, C_ch] float32 or None.  h_ckpt [b, L//s, H, P, N] and conv_ckpt
    [b, L//s, 3, C_ch] (the forward's checkpoints, s a multiple of 64) rebuild each cell
    of s tokens on its own; without them the whole sequence is rebuilt from h0, tail_in.
    """
    _cuda(u, conv_w, dt, A, D, dy, conv_bias, tail_in, h0, h_ckpt, conv_ckpt, dh_final, dtail_out, workspace)
    b, L, cch = u.shape
    assert cch == H * P + 2 * G * N, "u must hold x|B|C channels"
    dev = u.device
    o = dict(out or {})
    shapes = {"du": (b, L, cch), "dtail_in": (b, 3, cch), "dconv_w": (cch, 4), "dconv_bias": (cch,),
              "ddt": (b, L, H), "dA": (H,), "dD": (H,), "dh0": (b, H, P, N)}
    for k, shp in shapes.items():
        if k not in o:
            o[k] = torch.empty(shp, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(layer_backward_workspace_size(b, L, H, P, N, G, _dtype_code(u)), 1),
                                dtype=torch.uint8, device=dev)
    for t, n in ((conv_w, "conv_w"), (conv_bias, "conv_bias"), (dt, "dt"), (A, "A"), (D, "D"), (h0, "h0"),
                 (h_ckpt, "h_ckpt"), (dh_final, "dh_final"), (dtail_out, "dtail_out"),
                 *((o[k], k) for k in shapes if o[k] is not None)):
        _f32(t, n)
    a = LayerBwdArgs()
    a.dtype = _dtype_code(u); a.b = b; a.L = L; a.H = H; a.P = P; a.N = N; a.G = G
    a.s = s if h_ckpt is not None else 0
    a.u = u.data_ptr(); a.u_batch_stride = u.stride(0); a.u_row_stride = u.stride(1)
    a.conv_w = conv_w.data_ptr(); a.conv_bias = _vp_of(conv_bias); a.tail_in = _vp_of(tail_in)
    a.conv_ckpt = _vp_of(conv_ckpt)
    a.dt = dt.data_ptr(); a.A = A.data_ptr(); a.D = _vp_of(D); a.h0 = _vp_of(h0); a.h_ckpt = _vp_of(h_ckpt)
    dy3 = dy.reshape(b, L, -1) if dy.dim() == 4 else dy
    a.dy = dy3.data_ptr(); a.dy_batch_stride = dy3.stride(0); a.dy_row_stride = dy3.stride(1)
    a.dh_final = _vp_of(dh_final); a.dtail_out = _vp_of(dtail_out)
    a.du = o["du"].data_ptr(); a.dtail_in = _vp_of(o["dtail_in"]); a.dconv_w = o["dconv_w"].data_ptr()
    a.dconv_bias = _vp_of(o["dconv_bias"]); a.ddt = o["ddt"].data_ptr(); a.dA = o["dA"].data_ptr()
    a.dD = _vp_of(o["dD"]); a.dh0 = _vp_of(o["dh0"])
    a.workspace = workspace.data_ptr(); a.workspace_bytes = workspace.numel()
    _check(lib().ssd_layer_backward(ctypes.byref(a), _stream(stream)))
    return o


def _vp_of(t):
    return None if t is None else t.data_ptr()


def gated_rmsnorm(y, z, weight, eps=1e-5, group_size=0, out=None, stream=None):
    """out = rmsnorm(y * silu(z)) * weight over groups of ``group_size`` channels (0: all).

    y, z: [..., d] with the same leading shape, rows of d contiguous channels
    (z may be a column slice of a wider tensor); weight: [d] float32.
    """
    _cuda(y, z, weight, out)
    _f32(weight, "weight")
    d = y.shape[-1]
    y2 = y.reshape(-1, d)
    z2 = z.reshape(-1, d) if z.is_contiguous() else z.flatten(0, -2)
    if out is None:
        out = torch.empty_like(y)
    o2 = out.view(-1, d)
    if z2.dtype != y2.dtype or o2.dtype != y2.dtype:
        raise TypeError("y, z and out must share the I/O dtype")
    rc = lib().ssd_gated_rmsnorm_forward(_ptr(y2), y2.stride(0), _ptr(z2), z2.stride(0), _ptr(weight), float(eps),
                                         int(group_size), _ptr(o2), o2.stride(0), y2.shape[0], d, _dtype_code(y2),
                                         _stream(stream))
    _check(rc)
    return out
