"""The chunked form of the Mamba-2 SSD backward, written out in fp64 numpy,
equals the oracle's step-by-step adjoint ("Mamba", Part IV Stage 7 applied to
the Part V recurrence).

This is the decomposition the GPU backward computes, phase by phase:
  * per chunk of 64 steps, lc_t = A_h sum_{s<=t} Delta_s; the chunk maps
    U_k = sum_u e^{lc_end - lc_u} Delta_u x_u B_u^T and V_k = sum_t e^{lc_t} dout_t C_t^T;
  * the passes S_{k+1} = e^{lc_end} S_k + U_k (state entering each chunk) and
    Gc_{k-1} = e^{lc_end} Gc_k + V_k (adjoint at each chunk's last step), dh0;
  * per chunk, the products that give dx, dz, dB, dC, and the decay gradient
    dl_t = dL/dlc_t (row minus column sums of W[t,s] = e^{lc_t - lc_s} Delta_s
    (C_t.B_s)(dout_t.x_s), the read-out through S0, and <Gc, S_end>), from which
    dDelta_s = x_s.(G_s B_s) + A_h sum_{t>=s} dl_t and dA_h = sum_s Delta_s sum_{t>=s} dl_t.
Steps past the sequence end are padded with zeros (Delta = 0), as on the GPU.
The check pins the derivation, independently of floating-point kernels.
"""
import numpy as np
import pytest

import oracle

Q = 64


def _sp(v):
    return np.logaddexp(0.0, v)


def _sg(v):
    return 1.0 / (1.0 + np.exp(-v))


def chunked_ssd_bwd(x, dt, A, B, C, dy, D, z, bias, softplus, h0, dfinal):
    bsz, L, nh, P = x.shape
    ng, N = B.shape[2], B.shape[3]
    hpg = nh // ng
    K = (L + Q - 1) // Q
    out = dict(dx=np.zeros_like(x), ddt=np.zeros_like(dt), dz=np.zeros_like(x), dA=np.zeros(nh),
               dD=np.zeros(nh), ddt_bias=np.zeros(nh), dB=np.zeros_like(B), dC=np.zeros_like(C),
               dh0=np.zeros((bsz, nh, P, N)))
    for b in range(bsz):
        for h in range(nh):
            g = h // hpg

            def chunk(k):
                t0 = k * Q
                nv = min(Q, L - t0)
                v = np.zeros(Q)
                Dt = np.zeros(Q)
                X = np.zeros((Q, P))
                O = np.zeros((Q, P))
                F = np.zeros((Q, P))  # dz factor dy sigma(z)(1 + z(1 - sigma(z)))
                Bs = np.zeros((Q, N))
                Cs = np.zeros((Q, N))
                v[:nv] = dt[b, t0:t0 + nv, h] + bias[h]
                Dt[:nv] = _sp(v[:nv]) if softplus else v[:nv]
                X[:nv] = x[b, t0:t0 + nv, h]
                dyy = dy[b, t0:t0 + nv, h]
                if z is not None:
                    zz = z[b, t0:t0 + nv, h]
                    O[:nv] = dyy * zz * _sg(zz)
                    F[:nv] = dyy * _sg(zz) * (1 + zz * (1 - _sg(zz)))
                else:
                    O[:nv] = dyy
                Bs[:nv] = B[b, t0:t0 + nv, g]
                Cs[:nv] = C[b, t0:t0 + nv, g]
                lc = A[h] * np.cumsum(Dt)
                return t0, nv, v, Dt, X, O, F, Bs, Cs, lc

            U, V, dec = [], [], []
            for k in range(K):
                _, _, _, Dt, X, O, _, Bs, Cs, lc = chunk(k)
                U.append((X * (np.exp(lc[-1] - lc) * Dt)[:, None]).T @ Bs)
                V.append((O * np.exp(lc)[:, None]).T @ Cs)
                dec.append(np.exp(lc[-1]))
            S, s = [], (h0[b, h].copy() if h0 is not None else np.zeros((P, N)))
            for k in range(K):
                S.append(s.copy())
                s = dec[k] * s + U[k]
            Gc, gacc = [None] * K, (dfinal[b, h].copy() if dfinal is not None else np.zeros((P, N)))
            for k in range(K - 1, -1, -1):
                Gc[k] = gacc.copy()
                gacc = dec[k] * gacc + V[k]
            out["dh0"][b, h] = gacc
            for k in range(K):
                t0, nv, v, Dt, X, O, F, Bs, Cs, lc = chunk(k)
                le, S0, G = lc[-1], S[k], Gc[k]
                lower = np.tril(np.ones((Q, Q)))
                dcy = np.exp(np.minimum(lc[:, None] - lc[None, :], 0.0)) * lower
                CB, XD = Cs @ Bs.T, O @ X.T
                CBL, XDL = dcy * CB, dcy * XD
                W = CBL * Dt[None, :] * XD
                SC, BG = Cs @ S0.T, Bs @ G.T
                el, er = np.exp(lc), np.exp(le - lc)
                yp = (CBL * Dt[None, :]) @ X + el[:, None] * SC
                gb = CBL.T @ O + er[:, None] * BG
                dx = Dt[:, None] * gb + D[h] * O
                dz = (yp + D[h] * X) * F
                dB = Dt[:, None] * (XDL.T @ Cs) + (er * Dt)[:, None] * (X @ G)
                dC = (XDL * Dt[None, :]) @ Bs + el[:, None] * (O @ S0)
                x3 = er * Dt * (X * BG).sum(1)
                dl = W.sum(1) - W.sum(0) + el * (O * SC).sum(1) - x3
                dl[-1] += np.exp(le) * (G * S0).sum() + x3.sum()
                q = np.cumsum(dl[::-1])[::-1]
                dd = (X * gb).sum(1) + A[h] * q
                dv = dd * _sg(v) if softplus else dd
                out["dx"][b, t0:t0 + nv, h] = dx[:nv]
                out["dz"][b, t0:t0 + nv, h] = dz[:nv]
                out["ddt"][b, t0:t0 + nv, h] = dv[:nv]
                out["dB"][b, t0:t0 + nv, g] += dB[:nv]
                out["dC"][b, t0:t0 + nv, g] += dC[:nv]
                out["dA"][h] += (Dt * q).sum()
                out["dD"][h] += (O * X).sum()
                out["ddt_bias"][h] += dv[:nv].sum()
    if z is None:
        out["dz"] = None
    return out


@pytest.mark.parametrize("bsz,L,nh,ng,P,N,softplus,gate,state", [
    (2, 150, 4, 2, 8, 6, True, True, True),     # ragged last chunk, groups of 2, h0 and dfinal
    (1, 64, 3, 1, 4, 5, True, False, False),    # one full chunk, no gate, zero states
    (1, 1, 2, 2, 3, 4, True, True, True),       # one step
    (2, 130, 2, 1, 5, 3, False, True, True),    # softplus off (Delta = |dt|)
])
def test_chunked_adjoint_equals_the_oracle(bsz, L, nh, ng, P, N, softplus, gate, state):
    rng = np.random.default_rng(900 + L)
    x = rng.standard_normal((bsz, L, nh, P))
    dt = rng.standard_normal((bsz, L, nh)) * 0.5 - 1.0
    bias = rng.standard_normal(nh) * 0.3
    if not softplus:
        dt, bias = np.abs(dt), np.zeros(nh)
    A = -np.exp(rng.standard_normal(nh) * 0.5)
    B = rng.standard_normal((bsz, L, ng, N))
    C = rng.standard_normal((bsz, L, ng, N))
    D = rng.standard_normal(nh)
    z = rng.standard_normal((bsz, L, nh, P)) if gate else None
    h0 = rng.standard_normal((bsz, nh, P, N)) if state else None
    dfinal = rng.standard_normal((bsz, nh, P, N)) if state else None
    dy = rng.standard_normal((bsz, L, nh, P))
    ref = oracle.ssd_bwd(x, dt, A, B, C, dy, D=D, z=z, dt_bias=bias, dt_softplus=softplus, h0=h0,
                         dfinal=dfinal)
    got = chunked_ssd_bwd(x, dt, A, B, C, dy, D, z, bias, softplus, h0, dfinal)
    for k in ("dx", "dz", "ddt", "dB", "dC", "dA", "dD", "ddt_bias", "dh0"):
        if ref[k] is None:
            assert got[k] is None
            continue
        err = np.max(np.abs(got[k] - ref[k]) / (1.0 + np.abs(ref[k])))
        assert err < 1e-10, (k, err)
