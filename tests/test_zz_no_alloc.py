"""ss_fwd_noalloc: the forward scan for callers that cannot allocate device memory.

A host that must not call cudaMalloc while it runs (a decode loop that cannot
afford the device synchronisation, or a memory planner that owns every byte of
the GPU) cannot hand ss_fwd a workspace.  ss_fwd_noalloc takes the same inputs
and outputs but uses a scratch area built into the library.  These tests call
it through the C ABI twice in a row, on problems that take the chunk-parallel
path (the only path that needs scratch), and compare every output with
ss_fwd's on the same inputs (within the parity tolerance, and bit for bit).
They also check that a problem too large for the
built-in area is refused, with nothing enqueued.
"""
import ctypes

import pytest
import torch

from selective_state_space_11_b200 import inputs as gen
from selective_state_space_11_b200 import ops
from tolerances import TOL, assert_close

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 4 << 20  # SS_FWD_NOALLOC_SCRATCH_BYTES in include/ss.h


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(p, y, fs, ck):
    b, d, L = p["u"].shape
    return ops.lib().ss_fwd_noalloc(
        b, d, 16, L, ops._DTYPE[p["u"].dtype], _p(p["u"]), _p(p["delta"]), _p(p["z"]), _p(p["A"]),
        _p(p["B"]), _p(p["C"]), _p(p["D"]), _p(p["delta_bias"]), 1, _p(y), _p(fs), _p(ck),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("bsz,dim,L,dtype", [(1, 16, 32768, "f32"), (2, 40, 3001, "bf16"),
                                             (1, 2048, 65536, "bf16")])
def test_noalloc_matches_ss_fwd_on_two_calls_in_a_row(bsz, dim, L, dtype):
    path, nseg = ops.fwd_path(bsz, dim, L)
    assert path == 1 and nseg > 1  # chunk-parallel: the path that needs scratch
    need = ops.lib().ss_fwd_workspace_size(bsz, dim, 16, L)
    assert 0 < need <= SCRATCH_BYTES
    tol = TOL[(dtype, "fwd")]
    for call, seed in enumerate((501, 502)):  # different inputs: no stale scratch is reused
        p = {k: (None if v is None else v.cuda())
             for k, v in gen.make_inputs(bsz, dim, 16, L, dtype, seed, with_dy=False).items()}
        ry, rfs, rck = ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                                  delta_bias=p["delta_bias"])
        y = torch.full_like(ry, float("nan"))
        fs = torch.full_like(rfs, float("nan"))
        ck = torch.full_like(rck, float("nan"))
        st = _noalloc(p, y, fs, ck)
        assert st == 0, ops.lib().ss_last_error().decode()
        torch.cuda.synchronize()
        n = assert_close(gen.as_f64(y), gen.as_f64(ry), tol, f"y, call {call}")
        n += assert_close(gen.as_f64(fs), gen.as_f64(rfs), tol, f"final state, call {call}")
        n += assert_close(gen.as_f64(ck), gen.as_f64(rck), tol, f"checkpoints, call {call}")
        assert n == y.numel() + fs.numel() + ck.numel()
        # the same kernels on the same inputs: bit for bit, so a word left in the
        # scratch by the previous call cannot hide under the tolerance
        assert torch.equal(y, ry) and torch.equal(fs, rfs) and torch.equal(ck, rck), f"call {call}"


def test_noalloc_refuses_problems_beyond_its_scratch():
    # find a chunk-parallel shape whose scratch need exceeds the built-in area
    dim, L = next((d, L) for L in (640, 1280, 2560) for d in range(4000, 4800, 5)
                  if ops.fwd_path(1, d, L)[0] == 1
                  and ops.lib().ss_fwd_workspace_size(1, d, 16, L) > SCRATCH_BYTES)
    p = {k: (None if v is None else v.cuda())
         for k, v in gen.make_inputs(1, dim, 16, L, "f32", 503, with_dy=False).items()}
    y = torch.full_like(p["u"], float("nan"))
    st = _noalloc(p, y, None, None)
    assert st == 4  # SS_ERR_WORKSPACE
    assert b"scratch" in ops.lib().ss_last_error()
    torch.cuda.synchronize()
    assert torch.isnan(y).all()  # refused before anything ran


def test_per_channel_problems_need_no_scratch():
    p = {k: (None if v is None else v.cuda())
         for k, v in gen.make_inputs(2, 2400, 16, 130, "bf16", 504, with_dy=False).items()}
    assert ops.fwd_path(2, 2400, 130)[0] == 0
    ry, rfs, rck = ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                              delta_bias=p["delta_bias"])
    y, fs, ck = torch.empty_like(ry), torch.empty_like(rfs), torch.empty_like(rck)
    ops.ss_fwd_noalloc(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                       delta_bias=p["delta_bias"], out=(y, fs, ck))
    torch.cuda.synchronize()
    assert torch.equal(y, ry) and torch.equal(fs, rfs) and torch.equal(ck, rck)
