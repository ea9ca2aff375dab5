"""Pins for the CPU oracle: facts fixed by the mathematics, not by the oracle.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
an independent statement of the same quantity:
  * the quadratic (attention-like) form of the selective-state layer,
    y = (M o C B^T) X + D X + decay * C h0^T, evaluated by brute force;
  * closed forms: A = 0 (exact prefix sums), constant inputs (geometric
    series), a single impulse, B = 0 / C = 0 (pure skip connection);
  * linearity in x and in h0;
  * the causal conv1d + SiLU against torch's grouped conv1d and SiLU;
  * bfloat16 round-to-nearest-even against torch's conversion;
  * checkpoint indexing and bitwise split/resume from (state, conv tail),
    with the negative control that resuming without the conv tail differs.
The same functions are run against deliberately broken builds of the oracle
(test_oracle_mutants.py) to show that each plausible mistake is caught.
"""
import math

import numpy as np
import torch

import oracle

RNG = np.random.default_rng


def _inputs(rng, b, L, H, P, N, G=1, dt_range=(1e-3, 0.3), h0=True):
    x = rng.standard_normal((b, L, H * P)).astype(np.float32)
    B = rng.standard_normal((b, L, G * N)).astype(np.float32)
    C = rng.standard_normal((b, L, G * N)).astype(np.float32)
    dt = rng.uniform(*dt_range, size=(b, L, H)).astype(np.float32)
    A = (-np.exp(rng.uniform(0, math.log(16), size=H))).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    h0v = rng.standard_normal((b, H, P, N)) if h0 else None
    return x, B, C, dt, A, D, h0v


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def quadratic_form(x, B, C, dt, A, D, h0, H, P, G):
    """Brute-force SSD quadratic form for every (batch, head)."""
    b, L = x.shape[:2]
    N = B.shape[2] // G
    y = np.zeros((b, L, H, P))
    hf = np.zeros((b, H, P, N))
    for bi in range(b):
        for h in range(H):
            g = h * G // H
            X = x[bi, :, h * P:(h + 1) * P].astype(np.float64)
            Bm = B[bi, :, g * N:(g + 1) * N].astype(np.float64)
            Cm = C[bi, :, g * N:(g + 1) * N].astype(np.float64)
            d = dt[bi, :, h].astype(np.float64)
            a = float(A[h])
            M = np.zeros((L, L))
            for i in range(L):
                for j in range(i + 1):
                    M[i, j] = d[j] * math.exp(a * math.fsum(d[j + 1:i + 1]))
            decay0 = np.array([math.exp(a * math.fsum(d[:i + 1])) for i in range(L)])
            CB = Cm @ Bm.T
            yy = (M * CB) @ X + float(D[h]) * X
            if h0 is not None:
                yy += decay0[:, None] * (Cm @ h0[bi, h].astype(np.float64).T)
            y[bi, :, h] = yy
            st = (M[L - 1][:, None] * X).T @ Bm
            if h0 is not None:
                st += decay0[L - 1] * h0[bi, h]
            hf[bi, h] = st
    return y, hf


def pin_quadratic_form():
    rng = RNG(11)
    for (b, L, H, P, N, G) in [(1, 17, 2, 3, 5, 1), (2, 40, 4, 4, 3, 2), (1, 64, 1, 8, 8, 1)]:
        x, B, C, dt, A, D, h0 = _inputs(rng, b, L, H, P, N, G)
        out = oracle.scan(x, B, C, dt, A, D, h0, s=0, G=G)
        yq, hq = quadratic_form(x, B, C, dt, A, D, h0, H, P, G)
        assert _rel(out["y"], yq) < 1e-12, ("y", _rel(out["y"], yq))
        assert _rel(out["h_final"], hq) < 1e-12, ("h_final", _rel(out["h_final"], hq))


def pin_A_zero_prefix_sum():
    rng = RNG(12)
    b, L, H, P, N = 1, 48, 2, 3, 4
    x, B, C, dt, A, D, h0 = _inputs(rng, b, L, H, P, N)
    A = np.zeros_like(A)
    out = oracle.scan(x, B, C, dt, A, D, h0, s=0)
    for h in range(H):
        for t in [0, 1, 7, L - 1]:
            st = np.zeros((P, N))
            for p in range(P):
                for n in range(N):
                    terms = [float(h0[0, h, p, n])] + [
                        float(dt[0, j, h]) * float(x[0, j, h * P + p]) * float(B[0, j, n])
                        for j in range(t + 1)]
                    st[p, n] = math.fsum(terms)
            for p in range(P):
                yv = math.fsum([float(C[0, t, n]) * st[p, n] for n in range(N)]
                               + [float(D[h]) * float(x[0, t, h * P + p])])
                got = out["y"][0, t, h, p]
                assert abs(got - yv) <= 1e-12 * max(1.0, abs(yv)), (t, h, p, got, yv)
        assert _rel(out["h_final"][0, h], st) < 1e-13 or t != L - 1


def pin_constant_geometric():
    rng = RNG(13)
    L, P, N = 200, 3, 2
    xv = rng.standard_normal(P)
    Bv = rng.standard_normal(N)
    Cv = rng.standard_normal(N)
    c = 0.05
    Ah = -2.5
    Dh = 0.7
    h0 = rng.standard_normal((1, 1, P, N))
    x = np.tile(xv.astype(np.float32), (1, L, 1))
    B = np.tile(Bv.astype(np.float32), (1, L, 1))
    C = np.tile(Cv.astype(np.float32), (1, L, 1))
    dt = np.full((1, L, 1), c, dtype=np.float32)
    out = oracle.scan(x, B, C, dt, np.array([Ah], np.float32), np.array([Dh], np.float32), h0, s=0)
    cc = float(np.float32(c))
    xx = x[0, 0].astype(np.float64)
    BB = B[0, 0].astype(np.float64)
    CC = C[0, 0].astype(np.float64)
    a = math.exp(cc * Ah)
    for t in [0, 1, 5, 99, L - 1]:
        k = t + 1
        st = a ** k * h0[0, 0].astype(np.float64) + cc * (1 - a ** k) / (1 - a) * np.outer(xx, BB)
        yv = st @ CC + np.float32(Dh) * xx
        assert _rel(out["y"][0, t, 0], yv) < 1e-12, (t, _rel(out["y"][0, t, 0], yv))
    assert _rel(out["h_final"][0, 0], st) < 1e-12


def pin_skip_only():
    rng = RNG(14)
    b, L, H, P, N = 2, 30, 3, 4, 5
    x, B, C, dt, A, D, _ = _inputs(rng, b, L, H, P, N, h0=False)
    exp = (x.reshape(b, L, H, P).astype(np.float64) * D[None, None, :, None].astype(np.float64))
    out = oracle.scan(x, np.zeros_like(B), C, dt, A, D, None, s=0)
    assert np.array_equal(out["y"], exp)
    out = oracle.scan(x, B, np.zeros_like(C), dt, A, D, None, s=0)
    assert np.array_equal(out["y"], exp)


def pin_single_impulse():
    rng = RNG(15)
    b, L, H, P, N = 1, 40, 2, 3, 4
    _, B, C, dt, A, D, _ = _inputs(rng, b, L, H, P, N, h0=False)
    t0 = 9
    x = np.zeros((b, L, H * P), np.float32)
    x[0, t0] = rng.standard_normal(H * P).astype(np.float32)
    out = oracle.scan(x, B, C, dt, A, None, None, s=0)
    for h in range(H):
        for t in range(L):
            if t < t0:
                st = np.zeros((P, N))
            else:
                dec = math.exp(float(A[h]) * math.fsum(dt[0, t0 + 1:t + 1, h].astype(np.float64)))
                st = dec * float(dt[0, t0, h]) * np.outer(x[0, t0, h * P:(h + 1) * P].astype(np.float64),
                                                          B[0, t0].astype(np.float64))
            yv = st @ C[0, t].astype(np.float64)
            assert np.allclose(out["y"][0, t, h], yv, rtol=1e-12, atol=1e-300), (t, h)


def pin_linearity():
    rng = RNG(16)
    b, L, H, P, N = 1, 50, 2, 4, 3
    x1, B, C, dt, A, D, h0a = _inputs(rng, b, L, H, P, N)
    x2 = rng.standard_normal(x1.shape).astype(np.float32)
    h0b = rng.standard_normal(h0a.shape)
    # exact sums of two float32 values are not float32 in general; use small integers
    x1 = np.round(x1 * 8) / 8
    x2 = np.round(x2 * 8) / 8
    h0a = np.round(h0a * 8) / 8
    h0b = np.round(h0b * 8) / 8
    ya = oracle.scan(x1, B, C, dt, A, D, h0a, s=0)["y"]
    yb = oracle.scan(x2, B, C, dt, A, D, h0b, s=0)["y"]
    yab = oracle.scan(x1 + x2, B, C, dt, A, D, h0a + h0b, s=0)["y"]
    assert _rel(yab, ya + yb) < 1e-12
    y2 = oracle.scan(2 * x1, B, C, dt, A, D, 2 * h0a, s=0)["y"]
    assert _rel(y2, 2 * ya) < 1e-14


def _torch_conv(u, w, bias, tail):
    ut = torch.from_numpy(u.astype(np.float64))
    b, L, cch = ut.shape
    if tail is None:
        pre = torch.zeros(b, 3, cch, dtype=torch.float64)
    else:
        pre = torch.from_numpy(tail.astype(np.float64))
    seq = torch.cat([pre, ut], dim=1).transpose(1, 2)            # [b, cch, L+3]
    wt = torch.from_numpy(w.astype(np.float64)).unsqueeze(1)      # [cch, 1, 4]
    bt = None if bias is None else torch.from_numpy(bias.astype(np.float64))
    z = torch.nn.functional.conv1d(seq, wt, bt, groups=cch)       # [b, cch, L]
    return torch.nn.functional.silu(z).transpose(1, 2).numpy()


def pin_conv_torch():
    rng = RNG(17)
    for (b, L, cch, with_tail, with_bias) in [(1, 20, 5, False, False), (2, 33, 7, True, True),
                                              (1, 2, 3, True, False), (1, 1, 4, True, True)]:
        u = rng.standard_normal((b, L, cch)).astype(np.float32)
        w = rng.uniform(-0.5, 0.5, (cch, 4)).astype(np.float32)
        bias = rng.standard_normal(cch).astype(np.float32) if with_bias else None
        tail = rng.standard_normal((b, 3, cch)).astype(np.float32) if with_tail else None
        v, tail_out = oracle.conv(u, w, bias, tail, io_round="none")
        ref = _torch_conv(u, w, bias, tail)
        assert _rel(v, ref) < 1e-6, _rel(v, ref)          # v is stored as float32
        full = np.concatenate([tail if tail is not None else np.zeros((b, 3, cch), np.float32), u], 1)
        assert np.array_equal(tail_out, full[:, -3:])


def pin_conv_delta_weights():
    rng = RNG(18)
    u = rng.standard_normal((1, 25, 6)).astype(np.float32)
    w = np.zeros((6, 4), np.float32)
    w[:, 3] = 1.0
    v, _ = oracle.conv(u, w, None, None, io_round="none")
    ref = torch.nn.functional.silu(torch.from_numpy(u.astype(np.float64))).numpy()
    assert np.allclose(v, ref.astype(np.float32), rtol=0, atol=0) or _rel(v, ref) < 1e-7


def pin_bf16_rounding():
    rng = RNG(19)
    vals = np.concatenate([
        rng.standard_normal(2000) * 10.0 ** rng.integers(-30, 30, 2000),
        # exact ties between consecutive bf16 values (even and odd significands)
        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 2.0 + 2 ** -7, -1.0 - 2 ** -8,
                  1.5 + 2 ** -9 * 0.999, 1e-39, 3e-40, -7.1e-41, 3.39e38]),
    ])
    ours = oracle.round_bf16(vals)
    ref = torch.from_numpy(vals).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    # torch goes through float32 first; that double rounding can only differ on
    # values within float32 rounding of a bf16 tie -- none of the values above.
    assert np.array_equal(ours, ref), vals[ours != ref][:5]
    v, _ = oracle.conv(rng.standard_normal((1, 40, 8)).astype(np.float32),
                       rng.uniform(-0.5, 0.5, (8, 4)).astype(np.float32), io_round="bf16")
    rt = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(v, rt)


def pin_ckpt_indexing():
    rng = RNG(20)
    b, L, H, P, N, s = 2, 70, 2, 3, 4, 16
    x, B, C, dt, A, D, h0 = _inputs(rng, b, L, H, P, N)
    out = oracle.scan(x, B, C, dt, A, D, h0, s=s)
    assert out["h_ckpt"].shape == (b, L // s, H, P, N)
    for k in range(L // s):
        m = (k + 1) * s
        pre = oracle.scan(x[:, :m], B[:, :m], C[:, :m], dt[:, :m], A, D, h0, s=0)
        assert np.array_equal(out["h_ckpt"][:, k], pre["h_final"]), k
        _, hq = quadratic_form(x[:, :m], B[:, :m], C[:, :m], dt[:, :m], A, D, h0, H, P, 1)
        assert _rel(out["h_ckpt"][:, k], hq) < 1e-12


def _layer_inputs(rng, b, L, H, P, N):
    cch = H * P + 2 * N
    u = rng.standard_normal((b, L, cch)).astype(np.float32)
    w = rng.uniform(-0.5, 0.5, (cch, 4)).astype(np.float32)
    bias = rng.standard_normal(cch).astype(np.float32) * 0.1
    dt = rng.uniform(1e-3, 0.2, (b, L, H)).astype(np.float32)
    A = (-np.exp(rng.uniform(0, math.log(16), H))).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    h0 = rng.standard_normal((b, H, P, N))
    tail = rng.standard_normal((b, 3, cch)).astype(np.float32)
    return u, w, bias, dt, A, D, h0, tail


def pin_split_resume_bitwise():
    rng = RNG(21)
    b, L, H, P, N, s = 2, 96, 2, 4, 3, 16
    u, w, bias, dt, A, D, h0, tail = _layer_inputs(rng, b, L, H, P, N)
    kw = dict(H=H, P=P, N=N, s=s, io_round="bf16")
    full = oracle.layer(u, w, dt, A, D, bias, tail, h0, **kw)
    for m in [32, 37, 1, 2]:
        p1 = oracle.layer(u[:, :m], w, dt[:, :m], A, D, bias, tail, h0, **kw)
        p2 = oracle.layer(u[:, m:], w, dt[:, m:], A, D, bias, p1["tail_out"], p1["h_final"], **kw)
        assert np.array_equal(np.concatenate([p1["y"], p2["y"]], 1), full["y"]), m
        assert np.array_equal(p2["h_final"], full["h_final"]), m
        assert np.array_equal(np.concatenate([p1["v"], p2["v"]], 1), full["v"]), m
        assert np.array_equal(p2["tail_out"], full["tail_out"]), m
        assert np.array_equal(p1["tail_out"], np.concatenate([tail, u], 1)[:, m:m + 3]), m
        if m % s == 0:
            both = np.concatenate([p1["h_ckpt"], p2["h_ckpt"]], 1)
            assert np.array_equal(both, full["h_ckpt"]), m
    # resuming from a stored checkpoint reproduces the unsplit run
    m = 2 * s
    p2 = oracle.layer(u[:, m:], w, dt[:, m:], A, D, bias, u[:, m - 3:m], full["h_ckpt"][:, 1], **kw)
    assert np.array_equal(p2["y"], full["y"][:, m:])


def pin_resume_needs_conv_tail():
    """Negative control: resuming the conv without its 3-token buffer is wrong."""
    rng = RNG(22)
    b, L, H, P, N = 1, 40, 2, 4, 3
    u, w, bias, dt, A, D, h0, tail = _layer_inputs(rng, b, L, H, P, N)
    kw = dict(H=H, P=P, N=N, s=0, io_round="none")
    full = oracle.layer(u, w, dt, A, D, bias, tail, h0, **kw)
    m = 20
    p1 = oracle.layer(u[:, :m], w, dt[:, :m], A, D, bias, tail, h0, **kw)
    good = oracle.layer(u[:, m:], w, dt[:, m:], A, D, bias, p1["tail_out"], p1["h_final"], **kw)
    bad = oracle.layer(u[:, m:], w, dt[:, m:], A, D, bias, None, p1["h_final"], **kw)
    assert np.array_equal(good["y"], full["y"][:, m:])
    assert np.array_equal(bad["v"][:, 3:], full["v"][:, m + 3:])
    assert not np.allclose(bad["v"][:, :3], full["v"][:, m:m + 3], rtol=1e-3)
    assert _rel(bad["y"], full["y"][:, m:]) > 1e-4


def _scan_loss(x, B, C, dt, A, D, h0, dy, dhf, H, P, G):
    """The scalar sum(dy * y) + sum(dhf * h_final) through the forward oracle."""
    out = oracle.scan(x, B, C, dt, A, D, h0, s=0, H=H, P=P, G=G, want_ckpt=False)
    return float(np.sum(out["y"] * dy) + np.sum(out["h_final"] * dhf))


def _fd_grad(f, arr, rel_step=None, abs_step=2.0 ** -5):
    """Central differences of f with respect to every element of arr.

    float32 inputs are perturbed in float32 and divided by the step actually
    taken.  With rel_step the step scales with the element and the estimate is
    Richardson-extrapolated (error O(step^4)); without it the step is fixed,
    which is exact for inputs the loss is linear in.
    """
    g = np.zeros(arr.shape)
    for i in range(arr.size):
        def diff(step):
            up, dn = arr.copy(), arr.copy()
            up.flat[i] = arr.flat[i] + step
            dn.flat[i] = arr.flat[i] - step
            width = float(up.flat[i]) - float(dn.flat[i])
            return (f(up) - f(dn)) / width
        if rel_step is None:
            g.flat[i] = diff(abs_step)
        else:
            st = rel_step * abs(float(arr.flat[i]))
            g.flat[i] = (4.0 * diff(st / 2) - diff(st)) / 3.0
    return g


def pin_backward_finite_differences():
    """Every gradient of the reverse mode against central differences of the forward."""
    rng = RNG(30)
    b, L, H, P, N, G = 2, 7, 4, 2, 2, 2
    x, B, C, dt, A, D, h0 = _inputs(rng, b, L, H, P, N, G=G, dt_range=(0.05, 0.4))
    dy = rng.standard_normal((b, L, H, P))
    dhf = rng.standard_normal((b, H, P, N))
    args = dict(x=x, B=B, C=C, dt=dt, A=A, D=D, h0=h0)
    bw = oracle.scan_backward(x, B, C, dt, A, D, dy, h0=h0, dh_final=dhf, H=H, P=P, G=G)

    def loss_wrt(name):
        def f(v):
            kw = dict(args)
            kw[name] = v
            return _scan_loss(kw["x"], kw["B"], kw["C"], kw["dt"], kw["A"], kw["D"], kw["h0"],
                              dy, dhf, H, P, G)
        return f

    # the loss is linear in x, B, C, D and h0: fixed steps give exact differences
    for name, key in [("x", "dx"), ("B", "dB"), ("C", "dC"), ("D", "dD"), ("h0", "dh0")]:
        fd = _fd_grad(loss_wrt(name), args[name])
        got = bw[key]
        if name == "x":
            got = got.reshape(b, L, H * P)
        elif name in ("B", "C"):
            got = got.reshape(b, L, G * N)
        assert _rel(got, fd) < 1e-9, (name, _rel(got, fd))
    for name, key in [("dt", "ddt"), ("A", "dA")]:
        fd = _fd_grad(loss_wrt(name), args[name], rel_step=1e-2)
        assert _rel(bw[key], fd) < 1e-7, (name, _rel(bw[key], fd))


def pin_backward_cells_equal_full():
    """Recomputing each cell from its checkpoint gives bitwise the gradients of
    one pass that keeps every state, including a ragged last cell."""
    rng = RNG(31)
    b, L, H, P, N, s = 2, 37, 2, 3, 4, 8
    x, B, C, dt, A, D, h0 = _inputs(rng, b, L, H, P, N)
    dy = rng.standard_normal((b, L, H, P))
    dhf = rng.standard_normal((b, H, P, N))
    fwd = oracle.scan(x, B, C, dt, A, D, h0, s=s)
    full = oracle.scan_backward(x, B, C, dt, A, D, dy, h0=h0, dh_final=dhf)
    cells = oracle.scan_backward(x, B, C, dt, A, D, dy, h0=h0, h_ckpt=fwd["h_ckpt"], dh_final=dhf, s=s)
    for k in full:
        assert np.array_equal(full[k], cells[k]), k


def pin_backward_without_input():
    """B = 0 leaves h_t = exp(A cumsum(dt)) h0, whose gradients have closed forms."""
    rng = RNG(32)
    b, L, H, P, N = 2, 11, 2, 3, 4
    x, B, C, dt, A, D, h0 = _inputs(rng, b, L, H, P, N)
    B = np.zeros_like(B)
    dy = rng.standard_normal((b, L, H, P))
    dhf = rng.standard_normal((b, H, P, N))
    bw = oracle.scan_backward(x, B, C, dt, A, D, dy, h0=h0, dh_final=dhf)
    xh = x.reshape(b, L, H, P).astype(np.float64)
    assert np.array_equal(bw["dx"], D.astype(np.float64)[None, None, :, None] * dy)
    assert abs(bw["dD"] - np.einsum("blhp,blhp->h", dy, xh)).max() < 1e-12 * np.abs(dy).sum()
    Cd = C.astype(np.float64)
    dC = np.zeros((b, L, N))
    dh0 = np.zeros((b, H, P, N))
    ddt = np.zeros((b, L, H))
    dA = np.zeros(H)
    for bi in range(b):
        for h in range(H):
            cum = np.cumsum(dt[bi, :, h].astype(np.float64))
            e = np.exp(float(A[h]) * cum)
            # r_t = dLoss/d(decay_t) for the factor e_t that multiplies h0 in h_t
            r = np.array([dy[bi, t, h] @ h0[bi, h] @ Cd[bi, t] for t in range(L)])
            r[-1] += np.sum(dhf[bi, h] * h0[bi, h])
            for t in range(L):
                dC[bi, t] += e[t] * (dy[bi, t, h] @ h0[bi, h])
                dh0[bi, h] += e[t] * np.outer(dy[bi, t, h], Cd[bi, t])
            dh0[bi, h] += e[-1] * dhf[bi, h]
            re = r * e
            ddt[bi, :, h] = float(A[h]) * np.cumsum(re[::-1])[::-1]
            dA[h] += np.sum(cum * re)
    assert _rel(bw["dC"][:, :, 0], dC) < 1e-12
    assert _rel(bw["dh0"], dh0) < 1e-12
    assert _rel(bw["ddt"], ddt) < 1e-12
    assert _rel(bw["dA"], dA) < 1e-12


def pin_gated_norm_torch():
    """The gated RMS norm against torch's rms_norm of y * silu(z) in fp64, four groups of 8."""
    rng = RNG(40)
    y = rng.standard_normal((3, 5, 32)).astype(np.float32)
    z = (2 * rng.standard_normal((3, 5, 32))).astype(np.float32)
    w = rng.standard_normal(32).astype(np.float32)
    eps = 1e-2
    got = oracle.gated_rmsnorm(y, z, w, eps=eps, group=8)
    v = torch.from_numpy(y).double() * torch.nn.functional.silu(torch.from_numpy(z).double())
    ref = torch.nn.functional.rms_norm(v.reshape(3, 5, 4, 8), (8,), eps=eps).reshape(3, 5, 32)
    ref = (ref * torch.from_numpy(w).double()).numpy()
    assert _rel(got, ref) < 1e-7, _rel(got, ref)
    # one group over all channels
    got1 = oracle.gated_rmsnorm(y, z, w, eps=eps)
    ref1 = (torch.nn.functional.rms_norm(v, (32,), eps=eps) * torch.from_numpy(w).double()).numpy()
    assert _rel(got1, ref1) < 1e-7


def pin_gated_norm_invariants():
    """A closed gate gives zero; without eps the norm ignores a power-of-two scale of y;
    the normalised squares of a group average to ms / (ms + eps)."""
    rng = RNG(41)
    y = rng.standard_normal((4, 64)).astype(np.float32)
    z = rng.standard_normal((4, 64)).astype(np.float32)
    w = rng.uniform(0.5, 2.0, 64).astype(np.float32)
    assert np.array_equal(oracle.gated_rmsnorm(y, np.zeros_like(z), w, group=16), np.zeros_like(y))
    a = oracle.gated_rmsnorm(y, z, w, eps=0.0, group=16)
    b = oracle.gated_rmsnorm(4 * y, z, w, eps=0.0, group=16)
    assert np.array_equal(a, b)
    eps = 0.25
    out = oracle.gated_rmsnorm(y, z, w, eps=eps, group=16).astype(np.float64) / w
    v = y.astype(np.float64) * (z / (1 + np.exp(-z.astype(np.float64))))
    ms = (v.reshape(4, 4, 16) ** 2).mean(-1)
    got = (out.reshape(4, 4, 16) ** 2).mean(-1)
    assert np.abs(got - ms / (ms + eps)).max() < 1e-6


def _torch_layer_grads(u, w, bias, tail, dt, A, D, h0, dy, dhf, dto, H, P, N, G):
    """Gradients of sum(dy*y) + sum(dhf*h_final) + sum(dto*tail_out) for the layer written
    out in torch fp64 (grouped conv1d + silu, then the recurrence one token at a time), by
    torch's autograd."""
    f = lambda a: torch.tensor(np.asarray(a, dtype=np.float64), requires_grad=True)
    ut, wt, bt, tt, dtt, At, Dt, h0t = map(f, (u, w, bias, tail, dt, A, D, h0))
    b, L, cch = u.shape
    seq = torch.cat([tt, ut], 1)                                                  # [b, L+3, cch]
    z = torch.nn.functional.conv1d(seq.transpose(1, 2), wt.unsqueeze(1), bt, groups=cch)
    v = torch.nn.functional.silu(z).transpose(1, 2)                             # [b, L, cch]
    x = v[:, :, :H * P].reshape(b, L, H, P)
    grp = [(h * G) // H for h in range(H)]
    Bm = v[:, :, H * P:H * P + G * N].reshape(b, L, G, N)[:, :, grp]             # [b, L, H, N]
    Cm = v[:, :, H * P + G * N:].reshape(b, L, G, N)[:, :, grp]
    h = h0t
    ys = []
    for t in range(L):
        a = torch.exp(dtt[:, t] * At)                                             # [b, H]
        h = a[:, :, None, None] * h + dtt[:, t, :, None, None] * x[:, t, :, :, None] * Bm[:, t, :, None, :]
        ys.append((h * Cm[:, t, :, None, :]).sum(-1) + Dt[None, :, None] * x[:, t])
    y = torch.stack(ys, 1)
    loss = (y * torch.from_numpy(dy)).sum() + (h * torch.from_numpy(dhf)).sum() + \
        (seq[:, -3:] * torch.from_numpy(dto)).sum()
    loss.backward()
    return {"du": ut.grad.numpy(), "dtail_in": tt.grad.numpy(), "dw": wt.grad.numpy(),
            "dbias": bt.grad.numpy(), "ddt": dtt.grad.numpy(), "dA": At.grad.numpy(),
            "dD": Dt.grad.numpy(), "dh0": h0t.grad.numpy()}


def _layer_grad_inputs(rng, b, L, H, P, N, G):
    cch = H * P + 2 * G * N
    u = rng.standard_normal((b, L, cch)).astype(np.float32)
    w = rng.uniform(-0.5, 0.5, (cch, 4)).astype(np.float32)
    bias = (rng.standard_normal(cch) * 0.3).astype(np.float32)
    dt = rng.uniform(1e-2, 0.3, (b, L, H)).astype(np.float32)
    A = (-np.exp(rng.uniform(0, math.log(16), H))).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    h0 = rng.standard_normal((b, H, P, N))
    tail = rng.standard_normal((b, 3, cch)).astype(np.float32)
    dy = rng.standard_normal((b, L, H, P))
    dhf = rng.standard_normal((b, H, P, N))
    dto = rng.standard_normal((b, 3, cch))
    return u, w, bias, tail, dt, A, D, h0, dy, dhf, dto


def pin_layer_backward_torch_autograd():
    """Every gradient of the layer's reverse mode (conv and scan) against torch autograd of
    an independent fp64 torch statement of the same layer; two groups, and L < 3."""
    rng = RNG(40)
    for (b, L, H, P, N, G) in [(2, 23, 2, 3, 4, 1), (1, 17, 4, 2, 3, 2), (1, 2, 2, 2, 2, 1)]:
        u, w, bias, tail, dt, A, D, h0, dy, dhf, dto = _layer_grad_inputs(rng, b, L, H, P, N, G)
        got = oracle.layer_backward(u, w, dt, A, D, dy, bias=bias, tail_in=tail, h0=h0, dh_final=dhf,
                                    dtail_out=dto, H=H, P=P, N=N, G=G, io_round="none")
        ref = _torch_layer_grads(u, w, bias, tail, dt, A, D, h0, dy, dhf, dto, H, P, N, G)
        for k in ref:
            assert _rel(got[k], ref[k]) < 1e-10, (k, (b, L, H, P, N, G), _rel(got[k], ref[k]))


def pin_layer_backward_finite_differences():
    """Every gradient of the layer's reverse mode against central differences of the forward
    oracle (conv + SiLU, then the recurrence): Richardson-extrapolated for the inputs the loss
    is nonlinear in (u, the conv buffer, w, bias, dt, A), fixed steps for D and h0."""
    rng = RNG(43)
    b, L, H, P, N, G = 1, 9, 2, 2, 2, 1
    u, w, bias, tail, dt, A, D, h0, dy, dhf, dto = _layer_grad_inputs(rng, b, L, H, P, N, G)
    args = dict(u=u, w=w, bias=bias, tail=tail, dt=dt, A=A, D=D, h0=h0)
    got = oracle.layer_backward(u, w, dt, A, D, dy, bias=bias, tail_in=tail, h0=h0, dh_final=dhf,
                                dtail_out=dto, H=H, P=P, N=N, G=G, io_round="none")

    def loss_wrt(name):
        def f(v):
            kw = dict(args)
            kw[name] = v
            out = oracle.layer(kw["u"], kw["w"], kw["dt"], kw["A"], kw["D"], kw["bias"], kw["tail"], kw["h0"],
                               H=H, P=P, N=N, G=G, s=0, io_round="none", want_ckpt=False)
            return float(np.sum(out["y"] * dy) + np.sum(out["h_final"] * dhf) + np.sum(out["tail_out"] * dto))
        return f

    # the conv's inputs reach the loss through v, which the forward stores in float32: larger
    # steps keep that rounding out of the differences
    for name, key, step, tol in [("u", "du", 5e-2, 1e-4), ("tail", "dtail_in", 5e-2, 1e-4),
                                 ("w", "dw", 5e-2, 1e-4), ("bias", "dbias", 5e-2, 1e-4),
                                 ("dt", "ddt", 1e-2, 1e-6), ("A", "dA", 1e-2, 1e-6)]:
        fd = _fd_grad(loss_wrt(name), args[name], rel_step=step)
        assert _rel(got[key], fd) < tol, (name, _rel(got[key], fd))
    for name, key in [("D", "dD"), ("h0", "dh0")]:
        fd = _fd_grad(loss_wrt(name), args[name])
        assert _rel(got[key], fd) < 1e-6, (name, _rel(got[key], fd))


def _conv_ckpt_from_u(u, s):
    """The 3 rows of u before every checkpoint boundary: [b, L//s, 3, Cch]."""
    b, L, cch = u.shape
    n = L // s
    return np.stack([u[:, (k + 1) * s - 3:(k + 1) * s] for k in range(n)], 1) if n else \
        np.zeros((b, 0, 3, cch), np.float32)


def pin_layer_backward_cells_equal_full():
    """Rebuilding each cell of s tokens from its state checkpoint and its 3-row conv buffer
    gives bitwise the gradients of the full reverse mode (exact checkpoints from the
    forward oracle; f32 and bf16 rounding of v, a ragged last cell)."""
    rng = RNG(41)
    for (b, L, H, P, N, s, io) in [(2, 96, 2, 4, 3, 32, "f32"), (1, 100, 2, 3, 2, 16, "bf16"),
                                   (1, 66, 2, 2, 3, 32, "f32")]:
        u, w, bias, tail, dt, A, D, h0, dy, dhf, dto = _layer_grad_inputs(rng, b, L, H, P, N, 1)
        fwd = oracle.layer(u, w, dt, A, D, bias, tail, h0, H=H, P=P, N=N, s=s, io_round=io)
        kw = dict(bias=bias, tail_in=tail, h0=h0, dh_final=dhf, dtail_out=dto, H=H, P=P, N=N, s=s,
                  io_round=io)
        full = oracle.layer_backward(u, w, dt, A, D, dy, **kw)
        cells = oracle.layer_backward(u, w, dt, A, D, dy, h_ckpt=fwd["h_ckpt"],
                                      conv_ckpt=_conv_ckpt_from_u(u, s), **kw)
        for k in full:
            assert np.array_equal(full[k], cells[k]), (k, L, s)


def pin_layer_backward_needs_conv_buffer():
    """Negative control: cells rebuilt with the state checkpoints but without their conv
    buffers (zeros) give wrong gradients of u and w."""
    rng = RNG(42)
    b, L, H, P, N, s = 1, 64, 2, 3, 2, 16
    u, w, bias, tail, dt, A, D, h0, dy, dhf, dto = _layer_grad_inputs(rng, b, L, H, P, N, 1)
    fwd = oracle.layer(u, w, dt, A, D, bias, tail, h0, H=H, P=P, N=N, s=s, io_round="f32")
    kw = dict(bias=bias, tail_in=tail, h0=h0, dh_final=dhf, H=H, P=P, N=N, s=s, io_round="f32")
    good = oracle.layer_backward(u, w, dt, A, D, dy, h_ckpt=fwd["h_ckpt"], conv_ckpt=_conv_ckpt_from_u(u, s), **kw)
    bad = oracle.layer_backward(u, w, dt, A, D, dy, h_ckpt=fwd["h_ckpt"],
                                conv_ckpt=np.zeros((b, L // s, 3, H * P + 2 * N), np.float32), **kw)
    full = oracle.layer_backward(u, w, dt, A, D, dy, **kw)
    assert np.array_equal(good["du"], full["du"])
    assert _rel(bad["dw"], full["dw"]) > 1e-3 and _rel(bad["du"], full["du"]) > 1e-4


PINS = [pin_quadratic_form, pin_A_zero_prefix_sum, pin_constant_geometric, pin_skip_only,
        pin_single_impulse, pin_linearity, pin_conv_torch, pin_conv_delta_weights,
        pin_bf16_rounding, pin_ckpt_indexing, pin_split_resume_bitwise,
        pin_resume_needs_conv_tail, pin_backward_finite_differences, pin_backward_cells_equal_full,
        pin_backward_without_input, pin_gated_norm_torch, pin_gated_norm_invariants,
        pin_layer_backward_torch_autograd, pin_layer_backward_finite_differences,
        pin_layer_backward_cells_equal_full,
        pin_layer_backward_needs_conv_buffer]
