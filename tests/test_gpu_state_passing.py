"""State passing through the C ABI against the fp64 oracle: an initial state
h0 for the forward, and for the backward the gradient arriving at the final
state (dfinal) and the gradient of h0 (dh0).  Covers every forward path (one
channel per lane group, channel pairs, chunk-parallel) and both reverse walks,
and the split-sequence identity: pieces chained through h0 / dh0 reproduce the
one-call results.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_11_b200 import inputs as gen
from selective_state_space_11_b200 import ops
from tolerances import TOL, assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
f64 = gen.as_f64


def _case(bsz, dim, L, dtype, seed):
    p = gen.make_inputs(bsz, dim, 16, L, dtype, seed)
    h0 = gen.make_state(bsz, dim, 16, seed)
    df = gen.make_state(bsz, dim, 16, seed + 1)
    return p, h0, df


def _dev(p):
    return {k: (None if v is None else v.to(DEV)) for k, v in p.items()}


def _orc(p, h0, df):
    args = [f64(p[k]) for k in ("u", "delta", "A", "B", "C")]
    kw = dict(D=f64(p["D"]), z=f64(p["z"]), delta_bias=f64(p["delta_bias"]), h0=f64(h0))
    y, fs, ck = oracle.ss_fwd(*args, **kw)
    g = oracle.ss_bwd(*args, f64(p["dy"]), dfinal=f64(df), **kw)
    return y, fs, ck, g


def _gpu(pd, h0, df):
    kw = dict(D=pd["D"], z=pd["z"], delta_bias=pd["delta_bias"])
    y, fs, ck = ops.ss_fwd(pd["u"], pd["delta"], pd["A"], pd["B"], pd["C"], h0=h0, **kw)
    g = ops.ss_bwd(pd["u"], pd["delta"], pd["A"], pd["B"], pd["C"], pd["dy"], ck, h0=h0,
                   dfinal=df, **kw)
    return y, fs, ck, g


# (batch, dim, L, dtype): one channel per lane group; channel pairs (ragged
# d_inner); chunk-parallel forward with ragged segments
SHAPES = [(2, 64, 200, "f32"), (2, 2400, 130, "bf16"), (2, 9500, 70, "f32"),
          (1, 40, 64 * 37 + 5, "f32")]


@pytest.mark.parametrize("bsz,dim,L,dtype", SHAPES)
def test_fwd_bwd_with_state(bsz, dim, L, dtype):
    p, h0, df = _case(bsz, dim, L, dtype, 301 + L)
    ry, rfs, rck, rg = _orc(p, h0, df)
    y, fs, ck, g = _gpu(_dev(p), h0.to(DEV), df.to(DEV))
    tf, tg = TOL[(dtype, "fwd")], TOL[(dtype, "grad")]
    assert_close(f64(y), ry, tf, "y")
    assert_close(f64(fs), rfs, tf, "final_state")
    assert_close(f64(ck), rck, tf, "checkpoints")
    for k, rk in [("du", "du"), ("ddelta", "ddelta"), ("dz", "dz"), ("dA", "dA"), ("dB", "dB"),
                  ("dC", "dC"), ("dD", "dD"), ("ddelta_bias", "dbias"), ("dh0", "dh0")]:
        assert_close(f64(g[k]), rg[rk], tg, k)


def test_zero_state_matches_plain_calls():
    """h0 = 0 and dfinal = 0 give bitwise the results of the plain entry points."""
    p = _dev(gen.make_inputs(2, 300, 16, 333, "bf16", 311))
    z0 = torch.zeros(2, 300, 16, device=DEV)
    kw = dict(D=p["D"], z=p["z"], delta_bias=p["delta_bias"])
    y1, f1, c1 = ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], **kw)
    y2, f2, c2 = ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], h0=z0, **kw)
    assert torch.equal(y1, y2) and torch.equal(f1, f2) and torch.equal(c1, c2)
    g1 = ops.ss_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], p["dy"], c1, **kw)
    g2 = ops.ss_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], p["dy"], c2, h0=z0, dfinal=z0,
                    **kw)
    for k in g1:
        if g1[k] is not None:
            assert torch.equal(g1[k], g2[k]), k


@pytest.mark.parametrize("bsz,dim,L,cut,dtype", [(2, 64, 300, 128, "f32"), (2, 9500, 150, 70, "bf16")])
def test_split_sequence_chains(bsz, dim, L, cut, dtype):
    """Two pieces chained through final_state -> h0 and dh0 -> dfinal equal the
    one-call forward and backward."""
    p, h0, df = _case(bsz, dim, L, dtype, 331 + L)
    pd = _dev(p)
    h0d, dfd = h0.to(DEV), df.to(DEV)
    y, fs, ck, g = _gpu(pd, h0d, dfd)

    def piece(lo, hi):
        q = dict(pd)
        for k in ("u", "delta", "z", "B", "C", "dy"):
            q[k] = pd[k][..., lo:hi].contiguous()
        return q

    p1, p2 = piece(0, cut), piece(cut, L)
    y1, fs1, c1, _ = _gpu(p1, h0d, torch.zeros_like(dfd))
    kw = dict(D=pd["D"], delta_bias=pd["delta_bias"])
    y2, fs2, c2 = ops.ss_fwd(p2["u"], p2["delta"], p2["A"], p2["B"], p2["C"], z=p2["z"], h0=fs1,
                             **kw)
    g2 = ops.ss_bwd(p2["u"], p2["delta"], p2["A"], p2["B"], p2["C"], p2["dy"], c2, z=p2["z"],
                    h0=fs1, dfinal=dfd, **kw)
    g1 = ops.ss_bwd(p1["u"], p1["delta"], p1["A"], p1["B"], p1["C"], p1["dy"], c1, z=p1["z"],
                    h0=h0d, dfinal=g2["dh0"], **kw)
    tf, tg = TOL[(dtype, "fwd")], TOL[(dtype, "grad")]
    assert_close(f64(torch.cat([y1, y2], -1)), f64(y), tf, "split y")
    assert_close(f64(fs2), f64(fs), tf, "split final state")
    for k in ("du", "ddelta", "dz", "dB", "dC"):
        assert_close(f64(torch.cat([g1[k], g2[k]], -1)), f64(g[k]), tg, f"split {k}")
    for k in ("dA", "dD", "ddelta_bias"):
        assert_close(f64(g1[k] + g2[k]), f64(g[k]), tg, f"split {k}")
    assert_close(f64(g1["dh0"]), f64(g["dh0"]), tg, "split dh0")


def test_autograd_with_initial_and_last_state():
    """selective_scan_fn(h0=..., return_last_state=True): gradients reach h0 and
    flow back from the returned last state."""
    p, h0, df = _case(2, 24, 100, "f32", 341)
    pd = _dev(p)
    leaves = {k: pd[k].clone().requires_grad_(True) for k in ("u", "delta", "B", "C")}
    h0d = h0.to(DEV).requires_grad_(True)
    y, last = ops.selective_scan_fn(leaves["u"], leaves["delta"], pd["A"], leaves["B"],
                                    leaves["C"], D=pd["D"], z=pd["z"],
                                    delta_bias=pd["delta_bias"], delta_softplus=True, h0=h0d,
                                    return_last_state=True)
    (y * pd["dy"]).sum().backward(retain_graph=True)
    ry, rfs, _, rg = _orc(p, h0, torch.zeros_like(df))
    tg = TOL[("f32", "grad")]
    assert_close(f64(y.detach()), ry, TOL[("f32", "fwd")], "y")
    assert_close(f64(last.detach()), rfs, TOL[("f32", "fwd")], "last state")
    assert_close(f64(h0d.grad), rg["dh0"], tg, "dh0 via autograd")
    assert_close(f64(leaves["u"].grad), rg["du"], tg, "du via autograd")
    # the last state's gradient enters as dfinal
    for t in list(leaves.values()) + [h0d]:
        t.grad = None
    ((y * pd["dy"]).sum() + (last * df.to(DEV)).sum()).backward()
    _, _, _, rg2 = _orc(p, h0, df)
    assert_close(f64(h0d.grad), rg2["dh0"], tg, "dh0 with dfinal")
    assert_close(f64(leaves["delta"].grad), rg2["ddelta"], tg, "ddelta with dfinal")
