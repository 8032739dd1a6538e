"""Mamba-2 SSD backward through the C ABI against the fp64 oracle's adjoint,
whose gradients are pinned to finite differences of the oracle's forward and
to the S6 backward with scalar A."""
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
KEYS = ("dx", "ddt", "dz", "dB", "dC", "dA", "dD", "ddt_bias", "dh0")


@pytest.fixture(autouse=True, params=["tcgen05", "tcgen05-heads", "mma"])
def ssd_kernel(request, monkeypatch):
    """Every case runs with the chunk maps on tcgen05 (default), on tcgen05
    with each chunk-gradient CTA taking as many heads of a group as divide it
    (SS_SSD_HEADS_PER_CTA=max; by default small grids keep one head per CTA),
    and on the tf32 mma.sync kernel (SS_SSD_VARIANT=mma); the device fault word
    of the bounded waits must stay clear."""
    if request.param == "mma":
        monkeypatch.setenv("SS_SSD_VARIANT", "mma")
    else:
        monkeypatch.delenv("SS_SSD_VARIANT", raising=False)
    if request.param == "tcgen05-heads":
        monkeypatch.setenv("SS_SSD_HEADS_PER_CTA", "max")
    else:
        monkeypatch.delenv("SS_SSD_HEADS_PER_CTA", raising=False)
    assert ops.lib().ss_device_fault(1) == 0
    yield request.param
    assert ops.lib().ss_device_fault(1) == 0, "a bounded wait ran out"


def _problem(bsz, L, nh, ng, N, dtype, seed, with_state=True, **kw):
    q = gen.make_ssd_inputs(bsz, L, nh, 64, ng, N, dtype, seed, **kw)
    q["dy"] = gen.make_ssd_inputs(bsz, L, nh, 64, ng, N, dtype, seed + 1)["x"]
    if with_state:
        q["h0"] = gen.make_state(bsz * nh, 64, N, seed).view(bsz, nh, 64, N)
        q["dfinal"] = gen.make_state(bsz * nh, 64, N, seed + 2).view(bsz, nh, 64, N)
    else:
        q["h0"] = q["dfinal"] = None
    return q


def _gpu(q, softplus=True):
    d = {k: (None if v is None else v.to(DEV)) for k, v in q.items()}
    g = ops.ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["dy"], D=d["D"], z=d["z"],
                    dt_bias=d["dt_bias"], dt_softplus=softplus, h0=d["h0"], dfinal=d["dfinal"])
    torch.cuda.synchronize()
    return {k: (None if v is None else f64(v)) for k, v in g.items()}


def _ref(q, heads=None, softplus=True):
    o = {k: (None if v is None else f64(v)) for k, v in q.items()}
    sel = slice(None) if heads is None else heads
    hs = lambda v, ax: None if v is None else np.take(v, np.arange(v.shape[ax])[sel], axis=ax)
    r = oracle.ssd_bwd(hs(o["x"], 2), hs(o["dt"], 2), hs(o["A"], 0), o["B"], o["C"], hs(o["dy"], 2),
                       D=hs(o["D"], 0), z=hs(o["z"], 2), dt_bias=hs(o["dt_bias"], 0),
                       dt_softplus=softplus, h0=hs(o["h0"], 1), dfinal=hs(o["dfinal"], 1))
    if q["D"] is None:
        r["dD"] = None
    if q["dt_bias"] is None:
        r["ddt_bias"] = None
    return r


def _compare(g, r, tol, heads=None, keys=KEYS):
    sel = slice(None) if heads is None else heads
    axis = {"dx": 2, "ddt": 2, "dz": 2, "dA": 0, "dD": 0, "ddt_bias": 0, "dh0": 1}
    for k in keys:
        if r.get(k) is None:
            continue
        got = g[k]
        if k in axis and heads is not None:
            got = np.take(got, np.arange(got.shape[axis[k]])[sel], axis=axis[k])
        assert_close(got, r[k], tol, k)


@pytest.mark.parametrize("bsz,L,nh,ng,N,dtype", [
    (2, 200, 4, 2, 64, "bf16"), (1, 64 * 3 + 17, 2, 1, 128, "f16"), (2, 64, 3, 3, 128, "bf16"),
    (1, 1, 2, 1, 64, "bf16"), (3, 130, 6, 2, 128, "bf16"), (1, 64 * 5, 4, 1, 128, "bf16")])
def test_ssd_bwd(bsz, L, nh, ng, N, dtype):
    """Several chunks with a ragged tail, one step, one chunk, groups of 1 to 6 heads."""
    q = _problem(bsz, L, nh, ng, N, dtype, 701 + L)
    _compare(_gpu(q), _ref(q), TOL[(dtype, "grad")])


def test_ssd_bwd_without_gate_skip_bias_or_state():
    q = _problem(2, 150, 4, 2, 128, "bf16", 711, with_state=False, with_z=False, with_D=False,
                 with_bias=False)
    g = _gpu(q)
    assert g["dz"] is None
    _compare(g, _ref(q), TOL[("bf16", "grad")])


def test_ssd_bwd_softplus_off():
    """Delta = dt without softplus and without dt_bias (dt taken as |dt|, so that
    Delta >= 0 and the decays stay at most 1; the generated dt_bias is negative)."""
    q = _problem(2, 140, 4, 1, 64, "bf16", 721, with_bias=False)
    q["dt"] = q["dt"].abs()
    _compare(_gpu(q, softplus=False), _ref(q, softplus=False), TOL[("bf16", "grad")])


def test_ssd_bwd_is_deterministic():
    q = _problem(2, 300, 8, 2, 128, "bf16", 731)
    a, b = _gpu(q), _gpu(q)
    for k in KEYS:
        if a[k] is not None:
            assert np.array_equal(a[k], b[k]), k


def test_ssd_bwd_chained_pieces():
    """The gradient of a sequence split in two pieces chained through the state
    (piece 2 starts from piece 1's final state, piece 1 receives piece 2's dh0 as
    its dfinal) equals the gradient of one call (GPU only)."""
    q = {k: (None if v is None else v.to(DEV)) for k, v in _problem(2, 256, 4, 2, 64, "bf16", 741).items()}
    kw = dict(D=q["D"], dt_bias=q["dt_bias"])
    full = ops.ssd_bwd(q["x"], q["dt"], q["A"], q["B"], q["C"], q["dy"], z=q["z"], h0=q["h0"],
                       dfinal=q["dfinal"], **kw)
    cut = 100
    piece = lambda k, lo, hi: q[k][:, lo:hi].contiguous()
    _, f1 = ops.ssd_fwd(piece("x", 0, cut), piece("dt", 0, cut), q["A"], piece("B", 0, cut),
                        piece("C", 0, cut), z=piece("z", 0, cut), h0=q["h0"], **kw)
    g2 = ops.ssd_bwd(piece("x", cut, 256), piece("dt", cut, 256), q["A"], piece("B", cut, 256),
                     piece("C", cut, 256), piece("dy", cut, 256), z=piece("z", cut, 256), h0=f1,
                     dfinal=q["dfinal"], **kw)
    g1 = ops.ssd_bwd(piece("x", 0, cut), piece("dt", 0, cut), q["A"], piece("B", 0, cut),
                     piece("C", 0, cut), piece("dy", 0, cut), z=piece("z", 0, cut), h0=q["h0"],
                     dfinal=g2["dh0"], **kw)
    tol = TOL[("bf16", "grad")]
    for k in ("dx", "ddt", "dz", "dB", "dC"):
        assert_close(f64(torch.cat([g1[k], g2[k]], 1)), f64(full[k]), tol, "chained " + k)
    for k in ("dA", "dD", "ddt_bias"):
        assert_close(f64(g1[k] + g2[k]), f64(full[k]), tol, "chained " + k)
    assert_close(f64(g1["dh0"]), f64(full["dh0"]), tol, "chained dh0")


def test_ssd_bwd_mamba2_layer_full_size_sampled():
    """The Mamba-2 2.7b layer shape (4 x 4096, 80 heads of 64, ngroups 1, dstate
    128, bf16) in the launch the benchmark times: every per-head output of heads
    0, 41 and 79 against the oracle.  dB and dC sum over all 80 heads; they are
    checked on the same sequence with those three heads alone."""
    q = _problem(4, 4096, 80, 1, 128, "bf16", 1005, with_state=False)
    heads = [0, 41, 79]
    g = _gpu(q)
    r = _ref(q, heads=heads)
    tol = TOL[("bf16", "grad")]
    _compare(g, r, tol, heads=heads, keys=("dx", "ddt", "dz", "dA", "dD", "ddt_bias", "dh0"))
    sub = dict(q)
    for k, ax in (("x", 2), ("dt", 2), ("z", 2), ("dy", 2)):
        sub[k] = q[k][:, :, heads].contiguous()
    for k in ("A", "D", "dt_bias"):
        sub[k] = q[k][heads].contiguous()
    _compare(_gpu(sub), r, tol, keys=("dB", "dC"))


_GROUP_REF = {}


def test_ssd_bwd_full_length_one_head_group(ssd_kernel):
    """The 2.7b layer's geometry (batch 4, L 4096, dstate 128, bf16) with one
    group of 8 heads: by default each chunk-gradient CTA takes all 8 and sums
    their dB, dC in its accumulators, so every output, dB and dC included, is
    checked at full length against the oracle (computed once for all kernel
    variants)."""
    q = _problem(4, 4096, 8, 1, 128, "bf16", 1015, with_state=False)
    if "r" not in _GROUP_REF:
        _GROUP_REF["r"] = _ref(q)
    _compare(_gpu(q), _GROUP_REF["r"], TOL[("bf16", "grad")])


def test_ssd_bwd_validation():
    q = {k: (None if v is None else v.to(DEV)) for k, v in _problem(1, 16, 2, 1, 64, "bf16", 751).items()}
    with pytest.raises(ValueError):
        ops.ssd_bwd(q["x"].float(), q["dt"], q["A"], q["B"], q["C"], q["dy"])
    with pytest.raises(ops.SSError, match="UNSUPPORTED"):
        ops.ssd_bwd(q["x"][..., :32].contiguous(), q["dt"], q["A"], q["B"], q["C"],
                    q["dy"][..., :32].contiguous())
    # a workspace below ss_ssd_bwd_workspace_size is rejected before any launch
    x, dt, A, B, C, dy = (q[k] for k in ("x", "dt", "A", "B", "C", "dy"))
    dx, ddt, dA = torch.empty_like(x), torch.empty_like(dt), torch.empty_like(A)
    dB, dC = torch.empty(B.shape, device=DEV), torch.empty(C.shape, device=DEV)
    ws = torch.empty(256, device=DEV, dtype=torch.uint8)
    P = ops._ptr
    st = ops.lib().ss_ssd_bwd(1, 16, 2, 64, 1, 64, ops.SS_BF16, P(x), P(dt), P(A), P(B), P(C), None, None,
                              None, 1, None, P(dy), None, P(dx), P(ddt), P(dA), P(dB), P(dC), None, None,
                              None, None, P(ws), ws.numel(), None)
    assert ops.STATUS[st] == "SS_ERR_WORKSPACE"


def test_ssd_fn_autograd_matches_the_abi():
    """ssd_fn's gradients (through torch.autograd, with the final state in the
    loss) are exactly those of a direct ss_ssd_bwd call."""
    q = {k: (None if v is None else v.to(DEV)) for k, v in _problem(2, 150, 4, 2, 64, "bf16", 761).items()}
    leaves = {k: q[k].clone().requires_grad_(True) for k in ("x", "dt", "A", "B", "C", "D", "z", "dt_bias", "h0")}
    y, fs = ops.ssd_fn(leaves["x"], leaves["dt"], leaves["A"], leaves["B"], leaves["C"], D=leaves["D"],
                       z=leaves["z"], dt_bias=leaves["dt_bias"], h0=leaves["h0"], return_final_state=True)
    torch.autograd.backward([y, fs], [q["dy"], q["dfinal"]])
    g = ops.ssd_bwd(q["x"], q["dt"], q["A"], q["B"], q["C"], q["dy"], D=q["D"], z=q["z"],
                    dt_bias=q["dt_bias"], h0=q["h0"], dfinal=q["dfinal"])
    pairs = dict(x="dx", dt="ddt", A="dA", D="dD", z="dz", dt_bias="ddt_bias", h0="dh0")
    for k, gk in pairs.items():
        assert torch.equal(leaves[k].grad, g[gk]), k
    assert torch.equal(leaves["B"].grad, g["dB"].to(torch.bfloat16))
    assert torch.equal(leaves["C"].grad, g["dC"].to(torch.bfloat16))
