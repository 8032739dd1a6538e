"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics.

Each pin checks the oracle against something other than itself:
  * the unrolled closed form of the recurrence ("Mamba", stanleyjacob.dev,
    Part V "S6, and why selectivity forbids the convolution": the weight from
    position s to t is C_t Abar_t ... Abar_{s+1} Bbar_s);
  * the time-invariant special case, a causal convolution with kernel
    K_k = C Abar^k Bbar (same section, the S4 view), evaluated by np.convolve;
  * closed forms: the geometric series for N = 1, a cumulative sum for A = 0,
    the single-step case L = 1, hand-derived golden values (tests/golden);
  * invariants: u = 0 gives y = 0, linearity in u, prefill + decode steps ==
    one long forward ("mamba-metal" README, "Long-context prompts"; niverel-mamba,
    "Autoregressive decoding"), the last checkpoint is the final state;
  * central finite differences of the forward for every gradient ("Mamba, on a
    laptop GPU.", "Correct, not just consistent": check against finite
    differences too), and homogeneity identities of the adjoint.
The numpy formulas here are written independently of ss_oracle.c (different
forms of softplus / sigmoid, explicit double sums instead of a recurrence).

Every pin takes an ``Oracle`` instance so that tests/test_oracle_mutants.py can
run the same pins against deliberately broken copies of the oracle.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------- helpers --
def rand_problem(rng, b, d, n, L, z=True, D=True, bias=True, h0=False):
    p = dict(u=rng.standard_normal((b, d, L)), delta=rng.standard_normal((b, d, L)),
             A=-np.exp(rng.uniform(-1.0, 1.0, (d, n))),
             B=rng.standard_normal((b, n, L)), C=rng.standard_normal((b, n, L)))
    p["z"] = rng.standard_normal((b, d, L)) if z else None
    p["D"] = rng.uniform(0, 1, d) if D else None
    p["delta_bias"] = rng.uniform(-2.0, 0.5, d) if bias else None
    p["h0"] = rng.standard_normal((b, d, n)) if h0 else None
    return p


def np_softplus(x):
    return np.logaddexp(0.0, x)


def np_silu(z):
    return z * 0.5 * (1.0 + np.tanh(0.5 * z))


def np_delta(p, softplus):
    x = p["delta"] + (0.0 if p["delta_bias"] is None else p["delta_bias"][None, :, None])
    return np_softplus(x) if softplus else x


def closed_form(p, softplus=True):
    """y and all states from the unrolled double sum (no recurrence)."""
    u, A, B, C = p["u"], p["A"], p["B"], p["C"]
    b_, d_, L = u.shape
    n_ = A.shape[1]
    dt = np_delta(p, softplus)
    y = np.zeros((b_, d_, L))
    H = np.zeros((b_, d_, L, n_))
    for b in range(b_):
        for d in range(d_):
            for t in range(L):
                h = np.zeros(n_)
                for s in range(t + 1):
                    w = np.exp(A[d] * dt[b, d, s + 1:t + 1].sum())
                    h += w * dt[b, d, s] * B[b, :, s] * u[b, d, s]
                if p.get("h0") is not None:
                    h += np.exp(A[d] * dt[b, d, :t + 1].sum()) * p["h0"][b, d]
                H[b, d, t] = h
                out = float(C[b, :, t] @ h)
                if p["D"] is not None:
                    out += p["D"][d] * u[b, d, t]
                y[b, d, t] = out * (np_silu(p["z"][b, d, t]) if p["z"] is not None else 1.0)
    return y, H


def fwd(orc, p, softplus=True, **kw):
    return orc.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                      delta_bias=p["delta_bias"], delta_softplus=softplus,
                      h0=p.get("h0"), **kw)


def bwd(orc, p, dy, softplus=True, dfinal=None):
    return orc.ss_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"], z=p["z"],
                      delta_bias=p["delta_bias"], delta_softplus=softplus, h0=p.get("h0"),
                      dfinal=dfinal)


def close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    assert a.size > 0, f"{what}: nothing compared"
    err = np.abs(a - b) / (1.0 + np.abs(b))
    assert np.all(np.isfinite(a)), f"{what}: non-finite"
    assert err.max() <= tol, f"{what}: max scaled err {err.max():.3e} > {tol:.1e}"
    return a.size


# ------------------------------------------------------------ forward pins --
def pin_closed_form(orc):
    rng = np.random.default_rng(11)
    n = 0
    for flags in [dict(), dict(z=False), dict(D=False), dict(bias=False)]:
        for sp in (True, False):
            p = rand_problem(rng, 2, 3, 5, 11, **flags)
            if not sp:
                p["delta"] = np.abs(p["delta"]) * 0.3  # keep Delta >= 0 without softplus
                p["delta_bias"] = None
            y, fs, _ = fwd(orc, p, softplus=sp)
            yc, H = closed_form(p, softplus=sp)
            n += close(y, yc, 1e-12, f"closed-form y {flags} sp={sp}")
            n += close(fs, H[:, :, -1], 1e-12, "closed-form final state")
    # an initial state h0 decays by exp(A * cumulative Delta)
    p = rand_problem(rng, 2, 2, 4, 9, h0=True)
    y, fs, _ = fwd(orc, p)
    yc, H = closed_form(p)
    n += close(y, yc, 1e-12, "closed-form y with h0")
    n += close(fs, H[:, :, -1], 1e-12, "closed-form final with h0")
    return n


def pin_checkpoints(orc):
    rng = np.random.default_rng(12)
    p = rand_problem(rng, 1, 2, 3, 150)
    y, fs, ck = fwd(orc, p)
    _, H = closed_form(p)
    assert ck.shape == (1, 2, 3, 3)
    n = close(ck[:, :, 0], H[:, :, 63], 1e-11, "checkpoint 0 = state after step 63")
    n += close(ck[:, :, 1], H[:, :, 127], 1e-11, "checkpoint 1 = state after step 127")
    n += close(ck[:, :, 2], H[:, :, 149], 1e-11, "ragged last checkpoint = state after L-1")
    n += close(ck[:, :, -1], fs, 0.0, "last checkpoint == final state")
    return n


def pin_s4_convolution(orc):
    """B, C and Delta constant in time: y = (K * u + D u) SiLU(z), K_k = sum_n C Abar^k Bbar."""
    rng = np.random.default_rng(13)
    b_, d_, n_, L = 2, 3, 4, 23
    p = rand_problem(rng, b_, d_, n_, L)
    Bc = rng.standard_normal((b_, n_))
    Cc = rng.standard_normal((b_, n_))
    p["B"] = np.repeat(Bc[:, :, None], L, axis=2)
    p["C"] = np.repeat(Cc[:, :, None], L, axis=2)
    dl = rng.standard_normal((b_, d_))
    p["delta"] = np.repeat(dl[:, :, None], L, axis=2)
    y, _, _ = fwd(orc, p)
    n = 0
    for b in range(b_):
        for d in range(d_):
            dt = np_softplus(dl[b, d] + p["delta_bias"][d])
            abar = np.exp(dt * p["A"][d])
            K = np.array([np.sum(Cc[b] * abar ** k * dt * Bc[b]) for k in range(L)])
            conv = np.convolve(p["u"][b, d], K)[:L]
            ref = (conv + p["D"][d] * p["u"][b, d]) * np_silu(p["z"][b, d])
            n += close(y[b, d], ref, 1e-12, "S4 convolution view")
    return n


def pin_zero_input(orc):
    rng = np.random.default_rng(14)
    p = rand_problem(rng, 2, 3, 4, 70)
    p["u"] = np.zeros_like(p["u"])
    y, fs, ck = fwd(orc, p)
    assert y.size and not np.any(y) and not np.any(fs) and not np.any(ck), "u = 0 must give 0"
    return y.size


def pin_A_zero_cumsum(orc):
    rng = np.random.default_rng(15)
    p = rand_problem(rng, 2, 3, 4, 17)
    p["A"] = np.zeros_like(p["A"])
    y, fs, _ = fwd(orc, p)
    dt = np_delta(p, True)
    # h_t[n] = sum_{s<=t} Delta_s B_s[n] u_s  (cumulative sum, no decay)
    inc = dt[:, :, None, :] * p["B"][:, None, :, :] * p["u"][:, :, None, :]  # (b,d,n,L)
    H = np.cumsum(inc, axis=3)
    ys = np.einsum("bnt,bdnt->bdt", p["C"], H)
    ref = (ys + p["D"][None, :, None] * p["u"]) * np_silu(p["z"])
    n = close(y, ref, 1e-12, "A = 0 cumulative sum")
    n += close(fs, H[:, :, :, -1], 1e-12, "A = 0 final state")
    return n


def pin_L1(orc):
    rng = np.random.default_rng(16)
    p = rand_problem(rng, 3, 4, 5, 1)
    y, fs, ck = fwd(orc, p)
    dt = np_delta(p, True)[:, :, 0]
    cb = np.sum(p["C"][:, :, 0] * p["B"][:, :, 0], axis=1)  # (b,)
    ref = (dt * p["u"][:, :, 0] * cb[:, None] + p["D"][None] * p["u"][:, :, 0]) \
        * np_silu(p["z"][:, :, 0])
    n = close(y[:, :, 0], ref, 1e-13, "L = 1 closed form")
    n += close(fs, dt[:, :, None] * p["B"][:, None, :, 0] * p["u"][:, :, 0:1], 1e-13,
               "L = 1 state")
    assert ck.shape == (3, 4, 1, 5)
    return n


def pin_geometric(orc):
    """N = 1, constant a = exp(Delta A), b = Delta B u: h_t = b (1 - a^{t+1}) / (1 - a)."""
    L = 40
    dt, A, Bv, Cv, u = 0.37, -0.8, 1.3, -0.6, 0.9
    p = dict(u=np.full((1, 1, L), u), delta=np.full((1, 1, L), dt), A=np.array([[A]]),
             B=np.full((1, 1, L), Bv), C=np.full((1, 1, L), Cv), z=None, D=None,
             delta_bias=None)
    y, fs, _ = fwd(orc, p, softplus=False)
    a = math.exp(dt * A)
    bb = dt * Bv * u
    h = np.array([bb * (1 - a ** (t + 1)) / (1 - a) for t in range(L)])
    n = close(y[0, 0], Cv * h, 1e-13, "geometric series")
    n += close(fs[0, 0, 0], h[-1], 1e-13, "geometric final")
    return n


def pin_golden(orc):
    """Hand-derived worked examples stored under tests/golden/."""
    n = 0
    for name in sorted(os.listdir(GOLDEN)):
        if not name.startswith("hand_") or not name.endswith(".json"):
            continue
        with open(os.path.join(GOLDEN, name)) as f:
            g = json.load(f)
        inp = {k: (None if v is None else np.array(v, dtype=np.float64))
               for k, v in g["inputs"].items()}
        if g["kind"] == "fwd":
            y, fs, _ = orc.ss_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                  D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                                  delta_softplus=bool(g["delta_softplus"]))
            n += close(y, np.array(g["expected"]["y"]), 1e-14, name + " y")
            n += close(fs, np.array(g["expected"]["final_state"]), 1e-14, name + " state")
        elif g["kind"] == "state_update":
            st, y = orc.ss_state_update(inp["state"], inp["u"], inp["delta"], inp["A"],
                                        inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                                        delta_bias=inp["delta_bias"],
                                        delta_softplus=bool(g["delta_softplus"]))
            n += close(y, np.array(g["expected"]["y"]), 1e-14, name + " y")
            n += close(st, np.array(g["expected"]["state"]), 1e-14, name + " state")
        elif g["kind"] == "bwd":
            gr = orc.ss_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["dy"],
                            D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                            delta_softplus=bool(g["delta_softplus"]))
            for k, v in g["expected"].items():
                n += close(gr[k], np.array(v), 1e-14, f"{name} {k}")
    assert n > 0, "no golden fixture compared"
    return n


def pin_linearity(orc):
    rng = np.random.default_rng(17)
    p = rand_problem(rng, 2, 3, 4, 33)
    u1, u2 = p["u"], rng.standard_normal(p["u"].shape)
    y1, s1, _ = fwd(orc, dict(p, u=u1))
    y2, s2, _ = fwd(orc, dict(p, u=u2))
    y3, s3, _ = fwd(orc, dict(p, u=0.7 * u1 - 1.9 * u2))
    n = close(y3, 0.7 * y1 - 1.9 * y2, 1e-12, "linear in u")
    n += close(s3, 0.7 * s1 - 1.9 * s2, 1e-12, "state linear in u")
    return n


def pin_prefill_decode(orc):
    """fwd(L1) then k decode steps == fwd(L1 + k), for y and the state."""
    rng = np.random.default_rng(18)
    L1, k = 37, 6
    p = rand_problem(rng, 2, 3, 4, L1 + k)
    y_full, fs_full, _ = fwd(orc, p)
    pre = {key: (v[..., :L1] if key in ("u", "delta", "z", "B", "C") and v is not None else v)
           for key, v in p.items()}
    y_pre, st, _ = fwd(orc, pre)
    n = close(y_pre, y_full[..., :L1], 1e-13, "prefill prefix")
    for j in range(L1, L1 + k):
        st, yj = orc.ss_state_update(st, p["u"][..., j], p["delta"][..., j], p["A"],
                                     p["B"][..., j], p["C"][..., j], D=p["D"],
                                     z=p["z"][..., j], delta_bias=p["delta_bias"])
        n += close(yj, y_full[..., j], 1e-12, f"decode step {j}")
    n += close(st, fs_full, 1e-12, "decode final state")
    return n


# ----------------------------------------------------------- backward pins --
def _loss(orc, p, dy, softplus, dfinal=None):
    y, fs, _ = fwd(orc, p, softplus=softplus)
    extra = float(np.sum(dfinal * fs)) if dfinal is not None else 0.0
    return float(np.sum(dy * y)) + extra


def pin_fd_gradients(orc):
    """Central differences of <dy, y> (+ <dfinal, final state>) for every element
    of every input."""
    rng = np.random.default_rng(19)
    n = 0
    cases = [(dict(h0=True), True), (dict(z=False), True), (dict(), False),
             (dict(D=False, bias=False), True), (dict(h0=True, dfinal=True), True)]
    names = {"u": "du", "delta": "ddelta", "z": "dz", "A": "dA", "B": "dB", "C": "dC",
             "D": "dD", "delta_bias": "dbias", "h0": "dh0"}
    for flags, sp in cases:
        flags = dict(flags)
        want_df = flags.pop("dfinal", False)
        p = rand_problem(rng, 2, 2, 3, 6, **flags)
        if not sp:
            p["delta"] = np.abs(p["delta"]) * 0.3
            p["delta_bias"] = np.abs(p["delta_bias"]) * 0.1 if p["delta_bias"] is not None else None
        dy = rng.standard_normal(p["u"].shape)
        df = rng.standard_normal(p["u"].shape[:2] + (p["A"].shape[1],)) if want_df else None
        an = bwd(orc, p, dy, softplus=sp, dfinal=df)
        for key, gname in names.items():
            if key in ("D", "delta_bias") and p[key] is None:
                # gradient with respect to a zero parameter that was omitted
                p2 = dict(p)
                p2[key] = np.zeros(p["u"].shape[1])
                base = p2
            elif p.get(key) is None:
                continue
            else:
                base = p
            x = base[key]
            fd = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                hstep = 1e-6 * max(1.0, abs(x[idx]))
                xp = x.copy(); xp[idx] += hstep
                xm = x.copy(); xm[idx] -= hstep
                fd[idx] = (_loss(orc, dict(base, **{key: xp}), dy, sp, df)
                           - _loss(orc, dict(base, **{key: xm}), dy, sp, df)) / (2 * hstep)
            n += close(an[gname], fd, 2e-7, f"FD {gname} {flags} dfinal={want_df} sp={sp}")
    return n


def _piece(p, lo, hi, h0=None):
    q = dict(p)
    for k in ("u", "delta", "z", "B", "C"):
        if q.get(k) is not None:
            q[k] = np.ascontiguousarray(q[k][..., lo:hi])
    q["h0"] = h0
    return q


def pin_split_sequence(orc):
    """A sequence cut in two pieces: the forward of the second piece starts from
    the first piece's final state, and the backward of the first piece receives
    the second piece's dh0 as the gradient of its final state.  Both reproduce
    the one-piece forward and backward exactly (up to rounding)."""
    rng = np.random.default_rng(23)
    n = 0
    for L, cut in ((150, 64), (97, 40)):
        p = rand_problem(rng, 2, 3, 4, L, h0=True)
        dy = rng.standard_normal(p["u"].shape)
        df = rng.standard_normal(p["h0"].shape)
        y, fs, ck = fwd(orc, p)
        g = bwd(orc, p, dy, dfinal=df)
        p1 = _piece(p, 0, cut, p["h0"])
        y1, fs1, ck1 = fwd(orc, p1)
        p2 = _piece(p, cut, L, fs1)
        y2, fs2, ck2 = fwd(orc, p2)
        n += close(np.concatenate([y1, y2], axis=-1), y, 1e-12, f"split fwd y L={L}")
        n += close(fs2, fs, 1e-12, f"split final state L={L}")
        if cut % 64 == 0:
            n += close(np.concatenate([ck1, ck2], axis=2), ck, 1e-12, f"split checkpoints L={L}")
        g2 = bwd(orc, p2, np.ascontiguousarray(dy[..., cut:]), dfinal=df)
        g1 = bwd(orc, p1, np.ascontiguousarray(dy[..., :cut]), dfinal=g2["dh0"])
        for k in ("du", "ddelta", "dz", "dB", "dC"):
            n += close(np.concatenate([g1[k], g2[k]], axis=-1), g[k], 1e-11, f"split {k} L={L}")
        for k in ("dA", "dD", "dbias"):
            n += close(g1[k] + g2[k], g[k], 1e-11, f"split {k} L={L}")
        n += close(g1["dh0"], g["dh0"], 1e-11, f"split dh0 L={L}")
    return n


def pin_adjoint_identities(orc):
    """Homogeneity: y is linear in u, in (B, C-part) and in D, so <grad, x> = <dy, part of y>."""
    rng = np.random.default_rng(20)
    p = rand_problem(rng, 2, 5, 4, 90)
    dy = rng.standard_normal(p["u"].shape)
    y, _, _ = fwd(orc, p)
    g = bwd(orc, p, dy)
    gate = np_silu(p["z"])
    skip = p["D"][None, :, None] * p["u"] * gate
    n = close(np.sum(g["du"] * p["u"]), np.sum(dy * y), 1e-11, "<du,u> = <dy,y>")
    n += close(np.sum(g["dB"] * p["B"]), np.sum(dy * (y - skip)), 1e-11, "<dB,B> = <dy,C h gate>")
    n += close(np.sum(g["dC"] * p["C"]), np.sum(dy * (y - skip)), 1e-11, "<dC,C> = <dy,C h gate>")
    n += close(np.sum(g["dD"] * p["D"]), np.sum(dy * skip), 1e-11, "<dD,D> = <dy,D u gate>")
    n += close(g["dbias"], g["ddelta"].sum(axis=(0, 2)), 1e-12, "dbias = sum ddelta")
    # z enters only through the gate: dz = dy * out * SiLU'(z), out from an ungated run
    out, _, _ = fwd(orc, dict(p, z=None))
    s = 0.5 * (1 + np.tanh(0.5 * p["z"]))
    n += close(g["dz"], dy * out * (s + p["z"] * s * (1 - s)), 1e-12, "dz closed form")
    return n


# ------------------------------------------------------- conv1d (Stage 2) --
def _np_conv(x, w, bias, state_in, silu):
    """Causal depthwise conv as a library convolution: np.convolve of the window
    (incoming state, then x) with the reversed taps, keeping the L outputs."""
    bsz, dim, L = x.shape
    W = w.shape[1]
    u = np.empty_like(x)
    for b in range(bsz):
        for d in range(dim):
            pre_in = state_in[b, d] if state_in is not None else np.zeros(W - 1)
            seq = np.concatenate([pre_in, x[b, d]])
            pre = np.convolve(seq, w[d][::-1])[W - 1:W - 1 + L]
            if bias is not None:
                pre = pre + bias[d]
            u[b, d] = pre / (1.0 + np.exp(-pre)) if silu else pre
    return u


def pin_conv_library(orc):
    """conv1d against np.convolve, with and without SiLU, bias and incoming window;
    identity taps reproduce the input."""
    rng = np.random.default_rng(31)
    n = 0
    for W in (4, 2, 1):
        for silu in (False, True):
            x = rng.standard_normal((2, 3, 17))
            w = rng.standard_normal((3, W))
            bias = rng.standard_normal(3)
            st = rng.standard_normal((2, 3, W - 1))
            for b_, s_ in ((None, None), (bias, st)):
                u, so = orc.conv1d_fwd(x, w, bias=b_, state_in=s_, silu=silu)
                n += close(u, _np_conv(x, w, b_, s_, silu), 1e-12, f"conv W={W} silu={silu}")
                if W > 1:
                    win = np.concatenate([s_ if s_ is not None else np.zeros((2, 3, W - 1)), x], -1)
                    n += close(so, win[..., win.shape[-1] - (W - 1):], 0, f"conv state_out W={W}")
    x = rng.standard_normal((1, 2, 9))
    w = np.zeros((2, 4)); w[:, 3] = 1.0
    u, _ = orc.conv1d_fwd(x, w, silu=False)
    n += close(u, x, 0, "identity taps")
    return n


def pin_conv_pieces_and_decode(orc):
    """Pieces chained through state_out -> state_in, and token-by-token decode
    steps from a prefill's window, reproduce one full convolution."""
    rng = np.random.default_rng(32)
    x = rng.standard_normal((2, 3, 20))
    w = rng.standard_normal((3, 4))
    bias = rng.standard_normal(3)
    u, so = orc.conv1d_fwd(x, w, bias=bias, silu=True)
    n = 0
    for cut in (1, 2, 7, 19):
        u1, s1 = orc.conv1d_fwd(x[..., :cut].copy(), w, bias=bias, silu=True)
        u2, s2 = orc.conv1d_fwd(x[..., cut:].copy(), w, bias=bias, state_in=s1, silu=True)
        n += close(np.concatenate([u1, u2], -1), u, 1e-13, f"conv pieces cut={cut}")
        n += close(s2, so, 0, f"conv pieces state cut={cut}")
    _, st = orc.conv1d_fwd(x[..., :12].copy(), w, bias=bias, silu=True)
    for t in range(12, 20):
        st, ut = orc.conv1d_step(st, x[..., t].copy(), w, bias=bias, silu=True)
        n += close(ut, u[..., t], 1e-13, f"conv decode step {t}")
    n += close(st, so, 0, "conv decode final window")
    return n


def pin_conv_gradients(orc):
    """Central differences of <du, u> + <dstate_out, state_out> for every element of
    x, w, bias and the incoming window; pieces chained backwards through
    dstate_in -> dstate_out reproduce the one-call gradients."""
    rng = np.random.default_rng(33)
    n = 0
    for silu in (True, False):
        x = rng.standard_normal((2, 2, 7))
        w = rng.standard_normal((2, 4))
        bias = rng.standard_normal(2)
        st = rng.standard_normal((2, 2, 3))
        du = rng.standard_normal(x.shape)
        dso = rng.standard_normal(st.shape)
        g = orc.conv1d_bwd(x, w, du, bias=bias, state_in=st, silu=silu, dstate_out=dso)
        base = dict(x=x, w=w, bias=bias, state_in=st)

        def loss(q):
            u, so = orc.conv1d_fwd(q["x"], q["w"], bias=q["bias"], state_in=q["state_in"],
                                   silu=silu)
            return float(np.sum(du * u) + np.sum(dso * so))

        for key, gname in (("x", "dx"), ("w", "dw"), ("bias", "dbias"), ("state_in", "dstate_in")):
            v = base[key]
            fd = np.zeros_like(v)
            for idx in np.ndindex(v.shape):
                hstep = 1e-6 * max(1.0, abs(v[idx]))
                vp = v.copy(); vp[idx] += hstep
                vm = v.copy(); vm[idx] -= hstep
                fd[idx] = (loss(dict(base, **{key: vp})) - loss(dict(base, **{key: vm}))) / (2 * hstep)
            n += close(g[gname], fd, 2e-7, f"conv FD {gname} silu={silu}")
    # backward through two pieces
    x = rng.standard_normal((2, 3, 15))
    w = rng.standard_normal((3, 4))
    bias = rng.standard_normal(3)
    du = rng.standard_normal(x.shape)
    g = orc.conv1d_bwd(x, w, du, bias=bias, silu=True)
    cut = 6
    _, s1 = orc.conv1d_fwd(x[..., :cut].copy(), w, bias=bias, silu=True)
    g2 = orc.conv1d_bwd(x[..., cut:].copy(), w, du[..., cut:].copy(), bias=bias, state_in=s1,
                        silu=True)
    g1 = orc.conv1d_bwd(x[..., :cut].copy(), w, du[..., :cut].copy(), bias=bias, silu=True,
                        dstate_out=g2["dstate_in"])
    n += close(np.concatenate([g1["dx"], g2["dx"]], -1), g["dx"], 1e-12, "conv split dx")
    n += close(g1["dw"] + g2["dw"], g["dw"], 1e-12, "conv split dw")
    n += close(g1["dbias"] + g2["dbias"], g["dbias"], 1e-12, "conv split dbias")
    return n


# ------------------------------------------------------- seq_idx resets --
def seq_idx_cases(L, rng):
    """The nine structurally distinct packings of the niverel-mamba README's
    "seq_idx strict reset" (one row each), for a row length L >= 140."""
    def runs(lengths, first=0):
        ids = []
        for i, n in enumerate(lengths):
            ids += [first + i] * n
        return np.array(ids[:L] + [first + len(lengths)] * max(0, L - len(ids)), dtype=np.int32)
    cases = {
        "boundary_at_0": runs([L]),                      # one document from t = 0
        "length_1_docs": runs([1, 1, 5, 1, 30, 1]),
        "consecutive_boundaries": runs([10, 1, 1, 1, 40]),
        "boundary_on_chunk_edge": runs([64, 64]),
        "doc_inside_one_chunk": runs([70, 20]),
        "terminal_padding": np.where(np.arange(L) < L - 17, 0, -1).astype(np.int32),
        "nonzero_first_id": runs([50, 60], first=7),
        "many_short_docs": runs(list(rng.integers(1, 6, size=L))),
    }
    return cases


def _doc_runs(row):
    """[start, stop) of every maximal run of equal ids in a row."""
    cut = [0] + [t for t in range(1, len(row)) if row[t] != row[t - 1]] + [len(row)]
    return list(zip(cut[:-1], cut[1:]))


def pin_seq_idx(orc):
    """A packed row equals its documents run one by one from a zero state
    (forward and backward), for every packing case; rows of one batch are
    packed differently (misaligned across batch rows)."""
    rng = np.random.default_rng(41)
    L = 150
    cases = seq_idx_cases(L, rng)
    names = list(cases)
    n = 0
    for i0 in range(0, len(names), 3):
        group = names[i0:i0 + 3]
        bsz = len(group)
        p = rand_problem(rng, bsz, 3, 4, L)
        seq = np.stack([cases[g] for g in group])
        dy = rng.standard_normal(p["u"].shape)
        y, fs, _ = orc.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                              delta_bias=p["delta_bias"], seq_idx=seq)
        g = orc.ss_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"], z=p["z"],
                       delta_bias=p["delta_bias"], seq_idx=seq)
        acc = {k: np.zeros_like(g[k]) for k in ("dA", "dD", "dbias")}
        for b, name in enumerate(group):
            for lo, hi in _doc_runs(seq[b]):
                q = {k: (v[b:b + 1, ..., lo:hi].copy() if k in ("u", "delta", "z", "B", "C") else v)
                     for k, v in p.items() if k != "h0"}
                yd, fd, _ = orc.ss_fwd(q["u"], q["delta"], q["A"], q["B"], q["C"], D=q["D"],
                                       z=q["z"], delta_bias=q["delta_bias"])
                n += close(y[b:b + 1, :, lo:hi], yd, 1e-12, f"seq_idx y {name} [{lo},{hi})")
                if hi == L:
                    n += close(fs[b:b + 1], fd, 1e-12, f"seq_idx final state {name}")
                gd = orc.ss_bwd(q["u"], q["delta"], q["A"], q["B"], q["C"],
                                dy[b:b + 1, :, lo:hi].copy(), D=q["D"], z=q["z"],
                                delta_bias=q["delta_bias"])
                for k in ("du", "ddelta", "dz"):
                    n += close(g[k][b:b + 1, :, lo:hi], gd[k], 1e-11, f"seq_idx {k} {name}")
                for k in ("dB", "dC"):
                    n += close(g[k][b:b + 1, :, lo:hi], gd[k], 1e-11, f"seq_idx {k} {name}")
                for k in acc:
                    acc[k] += gd[k]
        for k in acc:
            n += close(g[k], acc[k], 1e-11, f"seq_idx {k} = sum over documents")
    return n


def pin_conv_seq_idx(orc):
    """Packed conv1d equals its documents convolved one by one (the first from
    the incoming window, the rest from a zero window), forward and backward."""
    rng = np.random.default_rng(42)
    L = 150
    cases = seq_idx_cases(L, rng)
    names = list(cases)
    n = 0
    for i0 in range(0, len(names), 4):
        group = names[i0:i0 + 4]
        bsz = len(group)
        x = rng.standard_normal((bsz, 3, L))
        w = rng.standard_normal((3, 4))
        bias = rng.standard_normal(3)
        st = rng.standard_normal((bsz, 3, 3))
        du = rng.standard_normal(x.shape)
        seq = np.stack([cases[g] for g in group])
        u, so = orc.conv1d_fwd(x, w, bias=bias, state_in=st, seq_idx=seq)
        g = orc.conv1d_bwd(x, w, du, bias=bias, state_in=st, seq_idx=seq)
        dw = np.zeros_like(w)
        db = np.zeros_like(bias)
        for b, name in enumerate(group):
            for lo, hi in _doc_runs(seq[b]):
                sin = st[b:b + 1] if lo == 0 else None
                ud, sd = orc.conv1d_fwd(x[b:b + 1, :, lo:hi].copy(), w, bias=bias, state_in=sin)
                n += close(u[b:b + 1, :, lo:hi], ud, 1e-12, f"conv seq_idx u {name}")
                if hi == L:
                    n += close(so[b:b + 1], sd, 0, f"conv seq_idx state_out {name}")
                gd = orc.conv1d_bwd(x[b:b + 1, :, lo:hi].copy(), w, du[b:b + 1, :, lo:hi].copy(),
                                    bias=bias, state_in=sin)
                n += close(g["dx"][b:b + 1, :, lo:hi], gd["dx"], 1e-12, f"conv seq_idx dx {name}")
                if lo == 0:
                    n += close(g["dstate_in"][b:b + 1], gd["dstate_in"], 1e-12,
                               f"conv seq_idx dstate_in {name}")
                dw += gd["dw"]
                db += gd["dbias"]
        n += close(g["dw"], dw, 1e-11, "conv seq_idx dw = sum over documents")
        n += close(g["dbias"], db, 1e-11, "conv seq_idx dbias = sum over documents")
    return n


# ------------------------------------------------------- Mamba-2 SSD --
def rand_ssd(rng, b, L, nh, P, ng, N, z=True, D=True, bias=True, h0=False):
    return dict(x=rng.standard_normal((b, L, nh, P)), dt=rng.standard_normal((b, L, nh)),
                A=-np.exp(rng.uniform(-1.0, 1.0, nh)),
                B=rng.standard_normal((b, L, ng, N)), C=rng.standard_normal((b, L, ng, N)),
                D=rng.uniform(0.0, 1.0, nh) if D else None,
                z=rng.standard_normal((b, L, nh, P)) if z else None,
                dt_bias=np.log(np.expm1(rng.uniform(1e-3, 0.1, nh))) if bias else None,
                h0=rng.standard_normal((b, nh, P, N)) if h0 else None)


def _ssd(orc, q, **kw):
    return orc.ssd_fwd(q["x"], q["dt"], q["A"], q["B"], q["C"], D=q["D"], z=q["z"],
                       dt_bias=q["dt_bias"], h0=q["h0"], **kw)


def pin_ssd_quadratic_form(orc):
    """The dual form: y = (L o (C B^T)) (Delta x) + decayed h0 read-out, with the
    semiseparable mask L[i,j] = exp(A sum_{k=j+1..i} Delta_k) for j <= i (the
    "masked quadratic attention" view), written with matrices, no recurrence."""
    rng = np.random.default_rng(51)
    n = 0
    for (nh, ng, h0) in ((4, 2, False), (3, 1, True), (2, 2, True)):
        q = rand_ssd(rng, 2, 37, nh, 5, ng, 6, h0=h0)
        y, fs = _ssd(orc, q)
        L = q["x"].shape[1]
        Dt = np_softplus(q["dt"] + q["dt_bias"][None, None, :])
        for b in range(2):
            for h in range(nh):
                g = h // (nh // ng)
                cs = np.cumsum(Dt[b, :, h]) * q["A"][h]
                mask = np.tril(np.exp(cs[:, None] - cs[None, :]))
                Bg, Cg = q["B"][b, :, g], q["C"][b, :, g]
                M = (Cg @ Bg.T) * mask * Dt[b, :, h][None, :]
                yq = M @ q["x"][b, :, h]
                if q["h0"] is not None:
                    yq += np.exp(cs)[:, None] * (Cg @ q["h0"][b, h].T)
                yq += q["D"][h] * q["x"][b, :, h]
                yq *= np_silu(q["z"][b, :, h])
                n += close(y[b, :, h], yq, 1e-11, f"SSD quadratic form nh={nh} ng={ng}")
                # final state from the same matrices: H_L = sum_j w_j x_j B_j^T (+ decayed h0)
                w = np.exp(cs[-1] - cs) * Dt[b, :, h]
                Hq = (q["x"][b, :, h] * w[:, None]).T @ Bg
                if q["h0"] is not None:
                    Hq += np.exp(cs[-1]) * q["h0"][b, h]
                n += close(fs[b, h], Hq, 1e-11, "SSD final state from the quadratic form")
    return n


def pin_ssd_is_scalar_a_s6(orc):
    """SSD with head h is S6 over the head's P channels with A[d, n] = A_h for all n,
    every channel sharing the head's Delta and the group's B, C."""
    rng = np.random.default_rng(52)
    q = rand_ssd(rng, 2, 40, 4, 3, 2, 5, h0=True)
    y, fs = _ssd(orc, q)
    n = 0
    for h in range(4):
        g = h // 2
        u = q["x"][:, :, h, :].transpose(0, 2, 1).copy()               # (b, P, L)
        delta = np.repeat(q["dt"][:, None, :, h], 3, axis=1)           # (b, P, L)
        A = np.full((3, 5), q["A"][h])
        B = q["B"][:, :, g, :].transpose(0, 2, 1).copy()               # (b, N, L)
        C = q["C"][:, :, g, :].transpose(0, 2, 1).copy()
        zz = q["z"][:, :, h, :].transpose(0, 2, 1).copy()
        ys, fss, _ = orc.ss_fwd(u, delta, A, B, C, D=np.full(3, q["D"][h]), z=zz,
                                delta_bias=np.full(3, q["dt_bias"][h]), h0=q["h0"][:, h])
        n += close(y[:, :, h, :].transpose(0, 2, 1), ys, 1e-12, f"SSD head {h} vs S6")
        n += close(fs[:, h], fss, 1e-12, f"SSD head {h} state vs S6")
    return n


def pin_ssd_split(orc):
    """Two pieces chained through the final state equal one call."""
    rng = np.random.default_rng(53)
    q = rand_ssd(rng, 2, 50, 2, 4, 1, 8, h0=True)
    y, fs = _ssd(orc, q)
    q1 = dict(q, **{k: q[k][:, :19].copy() for k in ("x", "dt", "B", "C", "z")})
    y1, f1 = _ssd(orc, q1)
    q2 = dict(q, **{k: q[k][:, 19:].copy() for k in ("x", "dt", "B", "C", "z")}, h0=f1)
    y2, f2 = _ssd(orc, q2)
    return close(np.concatenate([y1, y2], 1), y, 1e-12, "SSD split y") + \
        close(f2, fs, 1e-12, "SSD split state")


def _ssd_loss(orc, q, dy, df, sp):
    y, fs = orc.ssd_fwd(q["x"], q["dt"], q["A"], q["B"], q["C"], D=q["D"], z=q["z"],
                        dt_bias=q["dt_bias"], dt_softplus=sp, h0=q["h0"])
    return float(np.sum(dy * y)) + (float(np.sum(df * fs)) if df is not None else 0.0)


def _ssd_bwd(orc, q, dy, df, sp):
    return orc.ssd_bwd(q["x"], q["dt"], q["A"], q["B"], q["C"], dy, D=q["D"], z=q["z"],
                       dt_bias=q["dt_bias"], dt_softplus=sp, h0=q["h0"], dfinal=df)


def pin_ssd_fd_gradients(orc):
    """SSD backward: central differences of <dy, y> (+ <dfinal, final state>) for
    every element of every input, with grouped B/C, with and without softplus,
    gate, skip, bias and initial state."""
    rng = np.random.default_rng(54)
    names = {"x": "dx", "dt": "ddt", "A": "dA", "B": "dB", "C": "dC", "D": "dD", "z": "dz",
             "dt_bias": "ddt_bias", "h0": "dh0"}
    n = 0
    cases = [(2, 1, dict(h0=True), True, True), (4, 2, dict(), True, False),
             (2, 2, dict(z=False, D=False, bias=False), False, True)]
    for nh, ng, flags, sp, want_df in cases:
        q = rand_ssd(rng, 2, 5, nh, 2, ng, 3, **flags)
        if not sp:
            q["dt"] = np.abs(q["dt"]) * 0.3
        dy = rng.standard_normal(q["x"].shape)
        df = rng.standard_normal((2, nh, 2, 3)) if want_df else None
        an = _ssd_bwd(orc, q, dy, df, sp)
        for key, gname in names.items():
            if key in ("D", "dt_bias") and q[key] is None:
                base = dict(q, **{key: np.zeros(nh)})  # gradient at an omitted (zero) parameter
            elif key == "h0" and q["h0"] is None:
                base = dict(q, h0=np.zeros((2, nh, 2, 3)))
            elif q.get(key) is None:
                continue
            else:
                base = q
            v = base[key]
            fd = np.zeros_like(v)
            for idx in np.ndindex(v.shape):
                hstep = 1e-6 * max(1.0, abs(v[idx]))
                vp = v.copy(); vp[idx] += hstep
                vm = v.copy(); vm[idx] -= hstep
                fd[idx] = (_ssd_loss(orc, dict(base, **{key: vp}), dy, df, sp)
                           - _ssd_loss(orc, dict(base, **{key: vm}), dy, df, sp)) / (2 * hstep)
            n += close(an[gname], fd, 2e-7, f"SSD FD {gname} nh={nh} ng={ng} {flags} sp={sp}")
    return n


def pin_ssd_bwd_is_scalar_a_s6(orc):
    """The SSD backward equals the S6 backward of the same problem seen as S6
    (each head's P channels share the head's Delta, A[d, n] = A_h, the group's
    B and C): dx = du; ddt, dA_h, dD_h, ddt_bias_h = sums over the head's
    channels of ddelta, dA, dD, dbias; dB, dC of a group = S6 dB, dC over the
    group's channels; dz, dh0 unchanged."""
    rng = np.random.default_rng(55)
    bsz, L, nh, P, ng, N = 2, 30, 4, 3, 2, 5
    q = rand_ssd(rng, bsz, L, nh, P, ng, N, h0=True)
    dy = rng.standard_normal(q["x"].shape)
    df = rng.standard_normal((bsz, nh, P, N))
    an = _ssd_bwd(orc, q, dy, df, True)
    hpg = nh // ng
    n = 0
    for g in range(ng):
        hs = range(g * hpg, (g + 1) * hpg)
        # channels of the group's heads, head-major: channel (h, p)
        u = np.concatenate([q["x"][:, :, h, :].transpose(0, 2, 1) for h in hs], axis=1)
        delta = np.concatenate([np.repeat(q["dt"][:, None, :, h], P, axis=1) for h in hs], axis=1)
        A = np.concatenate([np.full((P, N), q["A"][h]) for h in hs])
        B = q["B"][:, :, g, :].transpose(0, 2, 1).copy()
        C = q["C"][:, :, g, :].transpose(0, 2, 1).copy()
        zz = np.concatenate([q["z"][:, :, h, :].transpose(0, 2, 1) for h in hs], axis=1)
        Dd = np.concatenate([np.full(P, q["D"][h]) for h in hs])
        bias = np.concatenate([np.full(P, q["dt_bias"][h]) for h in hs])
        h0 = np.concatenate([q["h0"][:, h] for h in hs], axis=1)
        dys = np.concatenate([dy[:, :, h, :].transpose(0, 2, 1) for h in hs], axis=1)
        dfs = np.concatenate([df[:, h] for h in hs], axis=1)
        r = orc.ss_bwd(np.ascontiguousarray(u), np.ascontiguousarray(delta), A, B, C,
                       np.ascontiguousarray(dys), D=Dd, z=np.ascontiguousarray(zz),
                       delta_bias=bias, h0=np.ascontiguousarray(h0),
                       dfinal=np.ascontiguousarray(dfs))
        for k, h in enumerate(hs):
            sl = slice(k * P, (k + 1) * P)
            n += close(an["dx"][:, :, h, :], r["du"][:, sl].transpose(0, 2, 1), 1e-12, f"SSD dx h{h}")
            n += close(an["dz"][:, :, h, :], r["dz"][:, sl].transpose(0, 2, 1), 1e-12, f"SSD dz h{h}")
            n += close(an["ddt"][:, :, h], r["ddelta"][:, sl].sum(axis=1), 1e-12, f"SSD ddt h{h}")
            n += close(an["dA"][h], r["dA"][sl].sum(), 1e-12, f"SSD dA h{h}")
            n += close(an["dD"][h], r["dD"][sl].sum(), 1e-12, f"SSD dD h{h}")
            n += close(an["ddt_bias"][h], r["dbias"][sl].sum(), 1e-12, f"SSD ddt_bias h{h}")
            n += close(an["dh0"][:, h], r["dh0"][:, sl], 1e-12, f"SSD dh0 h{h}")
        n += close(an["dB"][:, :, g, :], r["dB"].transpose(0, 2, 1), 1e-12, f"SSD dB group {g}")
        n += close(an["dC"][:, :, g, :], r["dC"].transpose(0, 2, 1), 1e-12, f"SSD dC group {g}")
    return n


ALL_PINS = [pin_closed_form, pin_checkpoints, pin_s4_convolution, pin_zero_input,
            pin_A_zero_cumsum, pin_L1, pin_geometric, pin_golden, pin_linearity,
            pin_prefill_decode, pin_fd_gradients, pin_adjoint_identities, pin_split_sequence,
            pin_conv_library, pin_conv_pieces_and_decode, pin_conv_gradients, pin_seq_idx,
            pin_conv_seq_idx, pin_ssd_quadratic_form, pin_ssd_is_scalar_a_s6, pin_ssd_split,
            pin_ssd_fd_gradients, pin_ssd_bwd_is_scalar_a_s6]
