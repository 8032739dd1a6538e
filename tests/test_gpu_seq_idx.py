"""Packed documents (seq_idx) through the C ABI against the fp64 oracle, whose
packed runs are pinned to the documents run one by one.  Every packing case
of the niverel-mamba README's "seq_idx strict reset" list, on every forward
path (one channel per lane group, channel pairs, chunk-parallel), both
reverse walks, and the conv1d window."""
import numpy as np
import pytest
import torch

import oracle
import pins
from selective_state_space_11_b200 import inputs as gen
from selective_state_space_11_b200 import ops
from tolerances import TOL, assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
f64 = gen.as_f64


def _seq(bsz, L, seed):
    """bsz rows, each packed differently (misaligned across batch rows)."""
    rng = np.random.default_rng(seed)
    cases = list(pins.seq_idx_cases(L, rng).values())
    return np.stack([cases[(seed + b) % len(cases)] for b in range(bsz)]).astype(np.int32)


def _check_scan(bsz, dim, L, dtype, seed, with_h0=False):
    p = gen.make_inputs(bsz, dim, 16, L, dtype, seed)
    seq = _seq(bsz, L, seed)
    h0 = gen.make_state(bsz, dim, 16, seed) if with_h0 else None
    pd = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    sd = torch.from_numpy(seq).to(DEV)
    kw = dict(D=pd["D"], z=pd["z"], delta_bias=pd["delta_bias"], seq_idx=sd,
              h0=h0.to(DEV) if h0 is not None else None)
    y, fs, ck = ops.ss_fwd(pd["u"], pd["delta"], pd["A"], pd["B"], pd["C"], **kw)
    g = ops.ss_bwd(pd["u"], pd["delta"], pd["A"], pd["B"], pd["C"], pd["dy"], ck, **kw)
    args = [f64(p[k]) for k in ("u", "delta", "A", "B", "C")]
    okw = dict(D=f64(p["D"]), z=f64(p["z"]), delta_bias=f64(p["delta_bias"]), seq_idx=seq,
               h0=f64(h0) if h0 is not None else None)
    ry, rfs, rck = oracle.ss_fwd(*args, **okw)
    rg = oracle.ss_bwd(*args, f64(p["dy"]), **okw)
    tf, tg = TOL[(dtype, "fwd")], TOL[(dtype, "grad")]
    assert_close(f64(y), ry, tf, "y")
    assert_close(f64(fs), rfs, tf, "final_state")
    assert_close(f64(ck), rck, tf, "checkpoints")
    for k, rk in [("du", "du"), ("ddelta", "ddelta"), ("dz", "dz"), ("dA", "dA"), ("dB", "dB"),
                  ("dC", "dC"), ("dD", "dD"), ("ddelta_bias", "dbias")]:
        assert_close(f64(g[k]), rg[rk], tg, k)
    if with_h0:
        assert_close(f64(g["dh0"]), rg["dh0"], tg, "dh0")


# every packing case appears in the 3-row and 8-row batches below
@pytest.mark.parametrize("bsz,dim,L,dtype", [(8, 40, 150, "f32"), (3, 64, 300, "bf16"),
                                             (2, 2400, 160, "bf16"), (2, 9500, 150, "f32"),
                                             (2, 9496, 152, "bf16")])
def test_scan_seq_idx(bsz, dim, L, dtype):
    _check_scan(bsz, dim, L, dtype, 501 + L + dim)


def test_scan_seq_idx_with_initial_state():
    _check_scan(3, 64, 200, "f32", 511, with_h0=True)


def test_scan_seq_idx_chunk_parallel():
    """Long rows on the chunk-parallel forward: documents start inside and on
    the edges of the segments."""
    L = 64 * 37 + 5
    path, nseg = ops.fwd_path(1, 40, L)
    assert path == 1 and nseg > 1
    _check_scan(1, 40, L, "f32", 521)
    _check_scan(2, 24, L, "f32", 522, with_h0=True)


@pytest.mark.parametrize("bsz,dim,L,dtype", [(8, 40, 150, "f32"), (3, 96, 256, "bf16")])
def test_conv1d_seq_idx(bsz, dim, L, dtype):
    c = gen.make_conv_inputs(bsz, dim, L, 4, dtype, 531 + L)
    seq = _seq(bsz, L, 531 + L)
    cd = {k: v.to(DEV) for k, v in c.items()}
    sd = torch.from_numpy(seq).to(DEV)
    u, so = ops.conv1d_fwd(cd["x"], cd["w"], bias=cd["bias"], state_in=cd["state"], seq_idx=sd,
                           state_out=True)
    g = ops.conv1d_bwd(cd["x"], cd["w"], cd["du"], bias=cd["bias"], state_in=cd["state"],
                       seq_idx=sd)
    ru, rso = oracle.conv1d_fwd(f64(c["x"]), f64(c["w"]), bias=f64(c["bias"]),
                                state_in=f64(c["state"]), seq_idx=seq)
    rg = oracle.conv1d_bwd(f64(c["x"]), f64(c["w"]), f64(c["du"]), bias=f64(c["bias"]),
                           state_in=f64(c["state"]), seq_idx=seq)
    tf, tg = TOL[(dtype, "fwd")], TOL[(dtype, "grad")]
    assert_close(f64(u), ru, tf, "u")
    assert_close(f64(so), rso, 0, "state_out")
    assert_close(f64(g["dx"]), rg["dx"], tg, "dx")
    assert_close(f64(g["dstate_in"]), rg["dstate_in"], tg, "dstate_in")
    assert_close(f64(g["dw"]), rg["dw"], tg, "dw")
    assert_close(f64(g["dbias"]), rg["dbias"], tg, "dbias")
