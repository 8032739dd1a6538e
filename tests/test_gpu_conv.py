"""Causal depthwise conv1d (+ SiLU) through the C ABI against the fp64 oracle:
forward with incoming / outgoing windows, backward (dx, dw, dbias, window
gradient), pieces chained through the window, token-by-token decode steps,
bitwise determinism, and the full Mamba-2.8b layer shape."""
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


def _dev(c):
    return {k: v.to(DEV) for k, v in c.items()}


def _check(bsz, dim, L, W, dtype, seed, with_state=True, silu=True, with_bias=True):
    c = gen.make_conv_inputs(bsz, dim, L, W, dtype, seed)
    cd = _dev(c)
    st = cd["state"] if with_state else None
    b = cd["bias"] if with_bias else None
    dso = torch.randn(bsz, dim, W - 1, device=DEV) if W > 1 else None
    u, so = ops.conv1d_fwd(cd["x"], cd["w"], bias=b, state_in=st, silu=silu, state_out=True)
    g = ops.conv1d_bwd(cd["x"], cd["w"], cd["du"], bias=b, state_in=st, silu=silu,
                       dstate_out=dso, want_dstate_in=True)
    ru, rso = oracle.conv1d_fwd(f64(c["x"]), f64(c["w"]), bias=f64(b) if b is not None else None,
                                state_in=f64(c["state"]) if with_state else None, silu=silu)
    rg = oracle.conv1d_bwd(f64(c["x"]), f64(c["w"]), f64(c["du"]),
                           bias=f64(b) if b is not None else None,
                           state_in=f64(c["state"]) if with_state else None, silu=silu,
                           dstate_out=f64(dso) if dso is not None else None)
    tf, tg = TOL[(dtype, "fwd")], TOL[(dtype, "grad")]
    assert_close(f64(u), ru, tf, "u")
    if W > 1:
        assert_close(f64(so), rso, 0, "state_out")
        assert_close(f64(g["dstate_in"]), rg["dstate_in"], tg, "dstate_in")
    assert_close(f64(g["dx"]), rg["dx"], tg, "dx")
    assert_close(f64(g["dw"]), rg["dw"], tg, "dw")
    if with_bias:
        assert_close(f64(g["dbias"]), rg["dbias"], tg, "dbias")


@pytest.mark.parametrize("W", [4, 3, 2, 1])
@pytest.mark.parametrize("bsz,dim,L,dtype", [(2, 64, 200, "f32"), (2, 33, 7, "f32"),
                                             (3, 96, 129, "bf16"), (1, 40, 1, "f32")])
def test_conv1d_fwd_bwd(bsz, dim, L, W, dtype):
    _check(bsz, dim, L, W, dtype, 401 + L + W)


@pytest.mark.parametrize("silu,with_state,with_bias", [(False, False, False), (True, False, True),
                                                       (False, True, True)])
def test_conv1d_flags(silu, with_state, with_bias):
    _check(2, 48, 100, 4, "f32", 411, with_state=with_state, silu=silu, with_bias=with_bias)


def test_conv1d_f16_and_vector_rows():
    _check(2, 64, 256, 4, "f16", 421)
    _check(2, 64, 256, 4, "bf16", 422)


def test_conv1d_pieces_and_decode_steps():
    """Pieces chained through the window, and decode steps continuing a prefill,
    equal one call over the whole sequence."""
    c = _dev(gen.make_conv_inputs(2, 64, 150, 4, "f32", 431))
    u, so = ops.conv1d_fwd(c["x"], c["w"], bias=c["bias"], state_out=True)
    cut = 37
    u1, s1 = ops.conv1d_fwd(c["x"][..., :cut].contiguous(), c["w"], bias=c["bias"], state_out=True)
    u2, s2 = ops.conv1d_fwd(c["x"][..., cut:].contiguous(), c["w"], bias=c["bias"], state_in=s1,
                            state_out=True)
    assert torch.equal(torch.cat([u1, u2], -1), u) and torch.equal(s2, so)
    _, st = ops.conv1d_fwd(c["x"][..., :100].contiguous(), c["w"], bias=c["bias"], state_out=True)
    for t in range(100, 150):
        ut = ops.conv1d_step(st, c["x"][..., t].contiguous(), c["w"], bias=c["bias"])
        assert_close(f64(ut), f64(u[..., t]), 1e-6, f"decode step {t}")
    assert torch.equal(st, so)


def test_conv1d_deterministic():
    c = _dev(gen.make_conv_inputs(4, 300, 333, 4, "bf16", 441))
    g1 = ops.conv1d_bwd(c["x"], c["w"], c["du"], bias=c["bias"])
    g2 = ops.conv1d_bwd(c["x"], c["w"], c["du"], bias=c["bias"])
    for k in ("dx", "dw", "dbias"):
        assert torch.equal(g1[k], g2[k]), k


def test_conv1d_autograd():
    c = _dev(gen.make_conv_inputs(2, 24, 90, 4, "f32", 451))
    x = c["x"].clone().requires_grad_(True)
    w = c["w"].clone().requires_grad_(True)
    b = c["bias"].clone().requires_grad_(True)
    u = ops.causal_conv1d_fn(x, w, b, True)
    (u * c["du"]).sum().backward()
    rg = oracle.conv1d_bwd(f64(c["x"]), f64(c["w"]), f64(c["du"]), bias=f64(c["bias"]))
    assert_close(f64(x.grad), rg["dx"], 1e-4, "dx")
    assert_close(f64(w.grad), rg["dw"], 1e-4, "dw")


def test_conv1d_mamba2p8b_layer_full_size():
    """The layer shape the benchmark uses (4 x 5120 x 4096, bf16), in full."""
    w = gen.WORKLOADS["mamba2.8b_layer"]
    c = gen.make_conv_inputs(w.batch, w.dim, w.seqlen, 4, w.dtype, w.seed)
    cd = _dev(c)
    u, _ = ops.conv1d_fwd(cd["x"], cd["w"], bias=cd["bias"])
    g = ops.conv1d_bwd(cd["x"], cd["w"], cd["du"], bias=cd["bias"])
    ru, _ = oracle.conv1d_fwd(f64(c["x"]), f64(c["w"]), bias=f64(c["bias"]))
    assert_close(f64(u), ru, TOL[("bf16", "fwd")], "u full size")
    rg = oracle.conv1d_bwd(f64(c["x"]), f64(c["w"]), f64(c["du"]), bias=f64(c["bias"]))
    assert_close(f64(g["dx"]), rg["dx"], TOL[("bf16", "grad")], "dx full size")
    assert_close(f64(g["dw"]), rg["dw"], TOL[("bf16", "grad")], "dw full size")
    assert_close(f64(g["dbias"]), rg["dbias"], TOL[("bf16", "grad")], "dbias full size")
