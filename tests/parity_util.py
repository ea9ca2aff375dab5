"""Shared helpers of the GPU parity tests (comparison metrics, device moves)."""
import numpy as np
import torch

TOL = {"f32": 1e-5, "bf16": 1e-2}


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def host(t):
    return t.detach().float().cpu().numpy()


def check_outputs(out, ref, tol, heads=None, what=("y", "h_final", "h_ckpt")):
    """relL2 of y, h_final, the checkpoint stack and every checkpoint on its own."""
    errs = {}
    for k in what:
        if ref.get(k) is None or out.get(k) is None:
            continue
        g = out[k]
        if heads is not None:
            if k == "y":
                g = g[:, :, heads]
            elif k == "h_final":
                g = g[:, heads]
            else:
                g = g[:, :, heads]
        g = host(g)
        errs[k] = rel_l2(g, ref[k])
        if k == "h_ckpt" and ref[k].shape[1] > 0:
            errs["h_ckpt_max_single"] = max(rel_l2(g[:, i], ref[k][:, i]) for i in range(ref[k].shape[1]))
    bad = {k: e for k, e in errs.items() if not e <= tol}
    assert not bad, f"relL2 above {tol}: {bad} (all: {errs})"
    return errs
