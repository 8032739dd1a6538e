"""Mamba-2 SSD forward through the C ABI against the fp64 oracle, whose
recurrence is pinned to the masked quadratic form and to S6 with scalar A."""
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


@pytest.fixture(autouse=True, params=["tcgen05", "mma"])
def ssd_kernel(request, monkeypatch):
    """Every case runs on both forward kernels: the tcgen05/TMEM/TMA one
    (default) and the warp-level mma.sync one (SS_SSD_VARIANT=mma).  After each
    case the device fault word of the bounded waits must be clear."""
    if request.param == "mma":
        monkeypatch.setenv("SS_SSD_VARIANT", "mma")
    else:
        monkeypatch.delenv("SS_SSD_VARIANT", raising=False)
    want = 1 if request.param == "mma" else 0  # SS_SSD_PATH_MMA, SS_SSD_PATH_TCGEN05
    assert ops.lib().ss_ssd_fwd_path() == want
    assert ops.lib().ss_device_fault(1) == 0
    yield request.param
    assert ops.lib().ss_device_fault(1) == 0, "a bounded wait ran out"


def _run(q, h0=None, heads=None):
    qd = {k: (None if v is None else v.to(DEV)) for k, v in q.items()}
    y, fs = ops.ssd_fwd(qd["x"], qd["dt"], qd["A"], qd["B"], qd["C"], D=qd["D"], z=qd["z"],
                        dt_bias=qd["dt_bias"], h0=h0.to(DEV) if h0 is not None else None)
    sel = slice(None) if heads is None else heads
    o = {k: (None if v is None else f64(v)) for k, v in q.items()}
    sub = dict(x=o["x"][:, :, sel], dt=o["dt"][:, :, sel], A=o["A"][sel], B=o["B"], C=o["C"],
               D=None if o["D"] is None else o["D"][sel], z=None if o["z"] is None else o["z"][:, :, sel],
               dt_bias=None if o["dt_bias"] is None else o["dt_bias"][sel])
    ry, rfs = oracle.ssd_fwd(sub["x"], sub["dt"], sub["A"], sub["B"], sub["C"], D=sub["D"], z=sub["z"],
                             dt_bias=sub["dt_bias"],
                             h0=None if h0 is None else f64(h0)[:, sel])
    return f64(y)[:, :, sel], f64(fs)[:, sel], ry, rfs


@pytest.mark.parametrize("bsz,L,nh,ng,N,dtype", [
    (2, 200, 4, 2, 64, "bf16"), (1, 64 * 3 + 17, 2, 1, 128, "f16"), (2, 64, 3, 3, 128, "bf16"),
    (1, 1, 2, 1, 64, "bf16"), (3, 130, 6, 2, 128, "bf16")])
def test_ssd_fwd(bsz, L, nh, ng, N, dtype):
    q = gen.make_ssd_inputs(bsz, L, nh, 64, ng, N, dtype, 601 + L)
    y, fs, ry, rfs = _run(q)
    tol = TOL[(dtype, "fwd")]
    assert_close(y, ry, tol, "y")
    assert_close(fs, rfs, tol, "final_state")


def test_ssd_fwd_initial_state_and_flags():
    q = gen.make_ssd_inputs(2, 150, 4, 64, 1, 128, "bf16", 611, with_z=False, with_D=False,
                            with_bias=False)
    h0 = gen.make_state(2 * 4, 64, 128, 611).view(2, 4, 64, 128)
    y, fs, ry, rfs = _run(q, h0=h0)
    assert_close(y, ry, TOL[("bf16", "fwd")], "y with h0")
    assert_close(fs, rfs, TOL[("bf16", "fwd")], "final state with h0")


def test_ssd_split_sequence():
    """Two pieces chained through the final state equal one call (GPU only)."""
    q = {k: (None if v is None else v.to(DEV)) for k, v in
         gen.make_ssd_inputs(2, 256, 4, 64, 2, 64, "bf16", 621).items()}
    kw = dict(D=q["D"], dt_bias=q["dt_bias"])
    y, fs = ops.ssd_fwd(q["x"], q["dt"], q["A"], q["B"], q["C"], z=q["z"], **kw)
    cut = 100
    piece = lambda k, lo, hi: q[k][:, lo:hi].contiguous()
    y1, f1 = ops.ssd_fwd(piece("x", 0, cut), piece("dt", 0, cut), q["A"], piece("B", 0, cut),
                         piece("C", 0, cut), z=piece("z", 0, cut), **kw)
    y2, f2 = ops.ssd_fwd(piece("x", cut, 256), piece("dt", cut, 256), q["A"], piece("B", cut, 256),
                         piece("C", cut, 256), z=piece("z", cut, 256), h0=f1, **kw)
    tol = TOL[("bf16", "fwd")]
    assert_close(f64(torch.cat([y1, y2], 1)), f64(y), tol, "split y")
    assert_close(f64(f2), f64(fs), tol, "split state")


def test_ssd_mamba2_layer_full_size_sampled():
    """The Mamba-2 2.7b layer shape (4 x 4096, 80 heads of 64, ngroups 1, dstate
    128, bf16) in the launch the benchmark times; heads 0, 41 and 79 checked
    against the oracle."""
    q = gen.make_ssd_inputs(4, 4096, 80, 64, 1, 128, "bf16", 1005)
    y, fs, ry, rfs = _run(q, heads=[0, 41, 79])
    tol = TOL[("bf16", "fwd")]
    assert_close(y, ry, tol, "y (sampled heads)")
    assert_close(fs, rfs, tol, "final state (sampled heads)")


def test_ssd_validation():
    q = {k: (None if v is None else v.to(DEV)) for k, v in
         gen.make_ssd_inputs(1, 16, 2, 64, 1, 64, "bf16", 631).items()}
    with pytest.raises(ValueError):
        ops.ssd_fwd(q["x"].float(), q["dt"], q["A"], q["B"], q["C"])
    with pytest.raises(ops.SSError, match="UNSUPPORTED"):
        ops.ssd_fwd(q["x"][..., :32].contiguous(), q["dt"], q["A"], q["B"], q["C"])


def test_bounded_wait_timeout_is_reported_and_the_context_recovers(ssd_kernel, monkeypatch):
    """SS_INJECT_WAIT_TIMEOUT makes the first chunk's copy wait of the tcgen05
    kernel run out on a barrier nothing arrives on: the kernel must set bit 0
    of the fault word, drain its copies and products, free its TMEM and
    return; the next call on the same context must be correct."""
    if ssd_kernel != "tcgen05":
        pytest.skip("the hook is in the tcgen05 kernel")
    q = gen.make_ssd_inputs(2, 200, 4, 64, 2, 64, "bf16", 641)
    qd = {k: (None if v is None else v.to(DEV)) for k, v in q.items()}
    monkeypatch.setenv("SS_INJECT_WAIT_TIMEOUT", "1")
    ops.ssd_fwd(qd["x"], qd["dt"], qd["A"], qd["B"], qd["C"], D=qd["D"], z=qd["z"], dt_bias=qd["dt_bias"])
    assert ops.lib().ss_device_fault(1) == 1  # bit 0 only; -1 would mean a CUDA error
    monkeypatch.delenv("SS_INJECT_WAIT_TIMEOUT")
    y, fs, ry, rfs = _run(q)
    assert_close(y, ry, TOL[("bf16", "fwd")], "y after the timeout")
    assert_close(fs, rfs, TOL[("bf16", "fwd")], "final state after the timeout")
