"""The chunked form of the backward pass, in fp64 numpy, against the oracle's reverse mode.

The CUDA backward evaluates the gradients chunk by chunk with closed forms
(state and adjoint chains over per-chunk summaries, and per-chunk products
with the decay matrix exp(cs_t - cs_j)); the formulas are stated in the
header of csrc/scan_bwd.cu.  This test writes those formulas out once more
with numpy, independently of the CUDA code, and checks them against the
oracle's token-by-token reverse mode on small shapes with a ragged last
chunk and cell, so that the algebra itself is pinned on the CPU.
"""
import numpy as np
import pytest

import oracle

Q = 64


def _chunked_backward(x, B, C, dt, A, D, dy, h0, dhf, h_ckpt, s, H, P, G):
    b, L = x.shape[:2]
    N = B.shape[2] // G
    nch = -(-L // Q)
    dx = np.zeros((b, L, H, P))
    dBh = np.zeros((b, L, H, N))
    dCh = np.zeros((b, L, H, N))
    ddt = np.zeros((b, L, H))
    dA = np.zeros(H)
    dD = np.zeros(H)
    dh0 = np.zeros((b, H, P, N))
    for bi in range(b):
        for h in range(H):
            g = h * G // H

            def chunk(c):
                t0 = c * Q
                r = min(Q, L - t0)
                X, Y, Bc, Cc, d = (np.zeros((Q, P)), np.zeros((Q, P)), np.zeros((Q, N)), np.zeros((Q, N)),
                                   np.zeros(Q))
                X[:r] = x[bi, t0:t0 + r, h * P:(h + 1) * P]
                Y[:r] = dy[bi, t0:t0 + r, h]
                Bc[:r] = B[bi, t0:t0 + r, g * N:(g + 1) * N]
                Cc[:r] = C[bi, t0:t0 + r, g * N:(g + 1) * N]
                d[:r] = dt[bi, t0:t0 + r, h]
                return t0, r, X, Y, Bc, Cc, d, np.cumsum(d * A[h])

            S, Gl, lam = [], [], []
            for c in range(nch):
                _, _, X, Y, Bc, Cc, d, cs = chunk(c)
                S.append((X * (d * np.exp(cs[-1] - cs))[:, None]).T @ Bc)
                Gl.append((Y * np.exp(cs)[:, None]).T @ Cc)
                lam.append(cs[-1])
            # states entering each chunk, restarted at every cell from its checkpoint
            cell = s // Q if h_ckpt is not None else nch
            hp = [None] * nch
            for k in range(-(-nch // cell)):
                hv = h0[bi, h] if k == 0 else h_ckpt[bi, k - 1, h]
                for c in range(k * cell, min(nch, (k + 1) * cell)):
                    hp[c] = hv
                    hv = np.exp(lam[c]) * hv + S[c]
            # adjoints reaching the last token of each chunk, from dh_final backwards
            gm = [None] * nch
            gv = dhf[bi, h]
            for c in range(nch - 1, -1, -1):
                gm[c] = gv
                gv = np.exp(lam[c]) * gv + Gl[c]
            dh0[bi, h] = gv
            for c in range(nch):
                t0, r, X, Y, Bc, Cc, d, cs = chunk(c)
                lm, Gam, hpv = cs[-1], gm[c], hp[c]
                CB, GX = Cc @ Bc.T, Y @ X.T
                seg = np.tril(np.exp(np.minimum(cs[:, None] - cs[None, :], 0.0)))
                K = np.tril(seg * GX * d[None, :] * CB, -1)
                CBm, GXm = seg * CB, seg * GX
                ecs, eend = np.exp(cs), np.exp(lm - cs)
                dxc = D[h] * Y + d[:, None] * (CBm.T @ Y + eend[:, None] * (Bc @ Gam.T))
                xg = X @ Gam
                dBr = GXm.T @ Cc + eend[:, None] * xg
                din = (Bc * dBr).sum(1)
                be = eend * d * (Bc * xg).sum(1)
                gh = Y @ hpv
                dCc = ecs[:, None] * gh + (GXm * d[None, :]) @ Bc
                al = ecs * (gh * Cc).sum(1)
                kp = np.concatenate([np.zeros((Q, 1)), np.cumsum(K, 1)[:, :-1]], 1)
                rr = np.array([kp[t:, t].sum() for t in range(Q)])
                term3 = np.exp(lm) * (Gam * hpv).sum()
                dl = np.array([al[t:].sum() + rr[t] + term3 + be[:t].sum() for t in range(Q)])
                dx[bi, t0:t0 + r, h] = dxc[:r]
                dBh[bi, t0:t0 + r, h] = (d[:, None] * dBr)[:r]
                dCh[bi, t0:t0 + r, h] = dCc[:r]
                ddt[bi, t0:t0 + r, h] = (A[h] * dl + din)[:r]
                dA[h] += (d * dl).sum()
                dD[h] += np.trace(GX)
    return {"dx": dx, "dB_h": dBh, "dC_h": dCh, "ddt": ddt, "dA": dA, "dD": dD, "dh0": dh0}


@pytest.mark.parametrize("L,s,G,ckpt", [(150, 64, 1, True), (200, 128, 2, True), (97, 64, 1, False)])
def test_chunk_formulas_match_reverse_mode(L, s, G, ckpt):
    rng = np.random.default_rng(L)
    b, H, P, N = 2, 2 * G, 3, 4
    x = rng.standard_normal((b, L, H * P)).astype(np.float32)
    B = rng.standard_normal((b, L, G * N)).astype(np.float32)
    C = rng.standard_normal((b, L, G * N)).astype(np.float32)
    dt = rng.uniform(0.01, 0.3, (b, L, H)).astype(np.float32)
    A = (-np.exp(rng.uniform(0, np.log(16), H))).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    h0 = rng.standard_normal((b, H, P, N))
    dy = rng.standard_normal((b, L, H, P))
    dhf = rng.standard_normal((b, H, P, N))
    fwd = oracle.scan(x, B, C, dt, A, D, h0, s=s, G=G)
    ref = oracle.scan_backward(x, B, C, dt, A, D, dy, h0=h0, dh_final=dhf, G=G)
    xd, Bd, Cd, dtd = (a.astype(np.float64) for a in (x, B, C, dt))
    got = _chunked_backward(xd, Bd, Cd, dtd, A.astype(np.float64), D.astype(np.float64), dy, h0, dhf,
                            fwd["h_ckpt"] if ckpt else None, s, H, P, G)
    for k in got:
        err = np.linalg.norm(got[k] - ref[k]) / np.linalg.norm(ref[k])
        assert err < 1e-12, (k, err)
