"""The reverse walk split into groups of 64-step chunks walked in parallel.

The gradient carry entering each group is composed from the later chunks'
maps c -> P_k c + e_k, formed in the states pass; the walk of every group then
starts from it.  These cases make the library pick more than one group (the
plan is read back through ss_bwd_path) on every walk variant, with every
optional input on (h0, dfinal, dh0, packed documents, z, D, bias), and check
all gradients against the fp64 oracle; plus run-to-run bit equality.  The
environment variable SS_BWD_VARIANT forces a variant, so the 4-lane walks are
also run on rows the one-channel-per-thread walk would take.
"""
import os

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


def _run(bsz, dim, L, dtype, seed, packed):
    p = gen.make_inputs(bsz, dim, 16, L, dtype, seed)
    h0 = gen.make_state(bsz, dim, 16, seed)
    df = gen.make_state(bsz, dim, 16, seed + 1)
    seq = None
    if packed:
        rng = np.random.default_rng(seed)
        cases = list(pins.seq_idx_cases(L, rng).values())
        seq = np.stack([cases[(seed + b) % len(cases)] for b in range(bsz)]).astype(np.int32)
    pd = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    sd = torch.from_numpy(seq).to(DEV) if packed else None
    kw = dict(D=pd["D"], z=pd["z"], delta_bias=pd["delta_bias"], h0=h0.to(DEV), seq_idx=sd)
    y, fs, ck = ops.ss_fwd(pd["u"], pd["delta"], pd["A"], pd["B"], pd["C"], **kw)
    g = ops.ss_bwd(pd["u"], pd["delta"], pd["A"], pd["B"], pd["C"], pd["dy"], ck,
                   dfinal=df.to(DEV), **kw)
    return p, h0, df, seq, g


@pytest.fixture
def force_variant():
    """Set SS_BWD_VARIANT for one test (None: the library's own choice)."""
    old = os.environ.get("SS_BWD_VARIANT")

    def _set(v):
        if v is None:
            os.environ.pop("SS_BWD_VARIANT", None)
        else:
            os.environ["SS_BWD_VARIANT"] = str(v)
    yield _set
    _set(old)


# (batch, dim, L, dtype, forced variant or None, expected variant): 16-byte
# aligned rows take the one-channel-per-thread walk (3); ragged rows one
# channel per lane group (0) or channel pairs (2); the 4-lane walks are also
# forced on aligned rows.  d_inner and the last chunk are ragged in several.
CASES = [(2, 64, 300, "f32", None, 3), (2, 64, 300, "f32", 0, 0),
         (3, 40, 64 * 9 + 7, "bf16", None, 0),
         (2, 1000, 64 * 10 + 3, "f32", None, 2), (2, 1016, 640, "bf16", None, 3),
         (2, 1016, 640, "bf16", 2, 2), (3, 200, 64 * 9 + 8, "bf16", None, 3)]


@pytest.mark.parametrize("bsz,dim,L,dtype,force,variant", CASES)
@pytest.mark.parametrize("packed", [False, True])
def test_grouped_walk_matches_oracle(bsz, dim, L, dtype, force, variant, packed, force_variant):
    force_variant(force)
    v, ng = ops.bwd_path(bsz, dim, L, dtype)
    assert v == variant and ng > 1, (v, ng)
    seed = 700 + L + dim + int(packed)
    p, h0, df, seq, g = _run(bsz, dim, L, dtype, seed, packed)
    args = [f64(p[k]) for k in ("u", "delta", "A", "B", "C")]
    okw = dict(D=f64(p["D"]), z=f64(p["z"]), delta_bias=f64(p["delta_bias"]), h0=f64(h0),
               seq_idx=seq)
    rg = oracle.ss_bwd(*args, f64(p["dy"]), dfinal=f64(df), **okw)
    tg = TOL[(dtype, "grad")]
    for k, rk in [("du", "du"), ("ddelta", "ddelta"), ("dz", "dz"), ("dA", "dA"), ("dB", "dB"),
                  ("dC", "dC"), ("dD", "dD"), ("ddelta_bias", "dbias"), ("dh0", "dh0")]:
        assert_close(f64(g[k]), rg[rk], tg, k)


def test_grouped_walk_is_deterministic():
    bsz, dim, L = 2, 1016, 640
    assert ops.bwd_path(bsz, dim, L, "bf16")[1] > 1
    g1 = _run(bsz, dim, L, "bf16", 731, True)[4]
    g2 = _run(bsz, dim, L, "bf16", 731, True)[4]
    for k in g1:
        if g1[k] is not None:
            assert torch.equal(g1[k], g2[k]), k


def test_layer_shapes_walk_in_groups():
    """Both layer shapes fill the GPU through chunk groups on the one-channel-
    per-thread walk."""
    for bsz, dim, L in [(4, 5120, 4096), (8, 1536, 2048)]:
        v, ng = ops.bwd_path(bsz, dim, L, "bf16")
        assert v == 3 and 1 < ng <= 32, (bsz, dim, L, v, ng)


def test_single_chunk_walks_in_one_group():
    assert ops.bwd_path(2, 64, 64, "f32")[1] == 1
    assert ops.bwd_path(4, 5120, 64, "bf16")[1] == 1
