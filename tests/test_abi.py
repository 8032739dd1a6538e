"""The C-ABI library loads and exports every symbol include/ss.h declares, and
host-side validation rejects bad arguments before anything touches a GPU."""
import ctypes
import os
import re

import pytest

import selective_state_space_11_b200.ops as ops
from selective_state_space_11_b200 import build as ssbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "ss.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(ss_[a-z_0-9]+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    ssbuild.build()
    return ops.lib()


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for s in ["ss_fwd", "ss_bwd", "ss_state_update", "ss_fwd_workspace_size",
              "ss_bwd_workspace_size", "ss_last_error", "ss_fwd_path", "ss_bwd_path"]:
        assert s in syms


def test_every_declared_symbol_is_exported(lib):
    syms = declared_symbols()
    assert syms
    for s in syms:
        assert hasattr(lib, s), f"{s} declared in ss.h but not exported"
        assert s in ops.SIGNATURES, f"{s} has no ctypes signature in the binding"


def test_only_abi_symbols_are_exported(lib):
    """-fvisibility=hidden: the library exports the C ABI and nothing of ours beyond it."""
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", ops.LIB_PATH], capture_output=True,
                         text=True).stdout
    ours = sorted({l.split()[-1] for l in out.splitlines() if " T " in l and "ss" in l.split()[-1]
                   and l.split()[-1].startswith("ss_")})
    assert ours == declared_symbols()


def test_version_and_status_strings(lib):
    assert lib.ss_version() >= 10000
    assert lib.ss_status_string(0) == b"SS_OK"
    assert lib.ss_status_string(4) == b"SS_ERR_WORKSPACE"
    assert lib.ss_status_string(99) == b"SS_UNKNOWN_STATUS"


def _fwd(lib, **kw):
    a = dict(batch=2, dim=4, dstate=16, seqlen=8, dtype=0, u=8, delta=8, z=None, A=16, B=8, C=8,
             D=None, bias=None, sp=1, y=8, fs=None, ck=None, ws=None, wsb=0, stream=None)
    a.update(kw)
    P = lambda v: None if v is None else ctypes.c_void_p(v)
    return lib.ss_fwd(a["batch"], a["dim"], a["dstate"], a["seqlen"], a["dtype"], P(a["u"]),
                      P(a["delta"]), P(a["z"]), P(a["A"]), P(a["B"]), P(a["C"]), P(a["D"]),
                      P(a["bias"]), a["sp"], P(a["y"]), P(a["fs"]), P(a["ck"]), P(a["ws"]),
                      a["wsb"], P(a["stream"]))


def test_validation_happens_before_any_cuda_call(lib):
    # None of these reach the device: they fail argument checks first.  The
    # pointer values are never dereferenced.
    assert _fwd(lib, batch=0) == 1
    assert _fwd(lib, seqlen=-3) == 1
    assert _fwd(lib, dstate=8) == 2
    assert b"dstate=8" in lib.ss_last_error()
    assert _fwd(lib, dtype=7) == 1
    assert _fwd(lib, u=None) == 1
    assert _fwd(lib, y=None) == 1
    assert _fwd(lib, u=9) == 3                     # fp32 data pointer not 4-byte aligned
    assert _fwd(lib, dtype=1, u=9) == 3            # bf16 pointer not 2-byte aligned
    assert _fwd(lib, fs=8) == 3                    # state outputs need 16-byte alignment
    assert _fwd(lib, batch=70000) == 2


def test_state_update_and_bwd_validation(lib):
    P = ctypes.c_void_p
    assert lib.ss_state_update(1, 4, 16, 0, None, P(16), P(16), None, P(16), P(16), P(16), None,
                               None, 1, P(16), None) == 1
    assert lib.ss_state_update(1, 4, 16, 0, P(8), P(16), P(16), None, P(16), P(16), P(16), None,
                               None, 1, P(16), None) == 3
    # z given without dz
    assert lib.ss_bwd(1, 4, 16, 8, 0, P(16), P(16), P(16), P(16), P(16), P(16), None, None, 1,
                      P(16), P(16), P(16), P(16), None, P(16), P(16), P(16), None, None,
                      P(16), 1 << 20, None) == 1
    # workspace too small is reported, not guessed around
    assert lib.ss_bwd(1, 4, 16, 8, 0, P(16), P(16), None, P(16), P(16), P(16), None, None, 1,
                      P(16), P(16), P(16), P(16), None, P(16), P(16), P(16), None, None,
                      P(16), 8, None) == 4
    assert b"workspace" in lib.ss_last_error()


def test_state_passing_validation(lib):
    """h0, dfinal and dh0 are fp32 states read and written 16 bytes at a time."""
    P = lambda v: None if v is None else ctypes.c_void_p(v)

    def fwd(h0):
        return lib.ss_fwd_with_state(2, 4, 16, 8, 0, P(16), P(16), None, P(16), P(16), P(16),
                                     None, None, 1, P(h0), None, P(16), None, None, None, 0, None)

    def bwd(h0=None, dfinal=None, dh0=None, seq=None):
        return lib.ss_bwd_with_state(1, 4, 16, 8, 0, P(16), P(16), None, P(16), P(16), P(16),
                                     None, None, 1, P(h0), P(seq), P(16), P(dfinal), P(16), P(16),
                                     P(16), None, P(16), P(16), P(16), None, None, P(dh0), P(16), 8,
                                     None)

    assert fwd(8) == 3
    assert b"state pointer" in lib.ss_last_error()
    assert bwd(h0=8) == 3 and bwd(dfinal=24) == 3 and bwd(dh0=4) == 3
    assert bwd(h0=32, dfinal=48, dh0=64) == 4   # aligned: reaches the workspace check
    assert bwd(seq=18) == 3 and b"seq_idx" in lib.ss_last_error()


def test_conv1d_validation(lib):
    P = lambda v: None if v is None else ctypes.c_void_p(v)

    def fwd(width=4, x=16, w=16, st=None, seq=None):
        return lib.ss_conv1d_fwd(2, 4, 8, width, 0, P(x), P(w), None, P(st), P(seq), 1, P(16), None,
                                 None)

    assert fwd(width=5) == 2 and b"width=5" in lib.ss_last_error()
    assert fwd(width=0) == 2
    assert fwd(x=None) == 1
    assert fwd(x=18) == 3                          # fp32 data pointer not 4-byte aligned
    assert fwd(st=6) == 3
    assert fwd(seq=2) == 3
    assert lib.ss_conv1d_bwd(2, 4, 8, 4, 0, P(16), P(16), None, None, None, 1, P(16), None, P(16),
                             P(16), None, None, P(16), 8, None) == 4
    assert lib.ss_conv1d_bwd_workspace_size(2, 4, 8, 9) == ctypes.c_size_t(-1).value
    assert lib.ss_conv1d_bwd_workspace_size(2, 4, 8, 4) >= 2 * 4 * 5 * 4
    assert lib.ss_conv1d_step(2, 4, 4, 0, None, P(16), P(16), None, 1, P(16), None) == 1


def test_bwd_workspace_size_is_pure_host_arithmetic(lib):
    """The size covers both reverse walks: the 4-lane walks (8-step states,
    16-channel block partials, up to 16 chunk groups) and the one-channel-per-
    thread walk (4-step states, 128-channel block partials, up to 32 groups)."""
    n = lib.ss_bwd_workspace_size(4, 5120, 16, 4096)
    nblk = (5120 + 15) // 16
    nchunk, groups = 4096 // 64, 16
    sub_states = 4 * 5120 * (4096 // 8) * 16 * 4
    partials = 2 * 4 * nblk * 16 * 4096 * 4 + groups * 4 * 5120 * (16 + 2) * 4
    chunk_maps = 2 * 4 * 5120 * nchunk * 16 * 4 + 4 * 5120 * groups * 16 * 4
    assert n >= sub_states + partials + chunk_maps
    ncb, chg = (5120 + 127) // 128, 32
    ch = (4 * 5120 * (4096 // 4) * 16 * 4 + 2 * 4 * ncb * 4096 * 16 * 4
          + chg * 4 * 5120 * (16 + 2) * 4 + 2 * 4 * nchunk * 5120 * 16 * 4 + 4 * chg * 5120 * 16 * 4)
    assert n >= ch
    # one chunk: a single group, so no carry maps for either walk
    one = lib.ss_bwd_workspace_size(4, 5120, 16, 64)
    old_one = 4 * 5120 * 8 * 16 * 4 + 2 * 4 * nblk * 16 * 64 * 4 + 4 * 5120 * 18 * 4
    ch_one = 4 * 5120 * 16 * 16 * 4 + 2 * 4 * ncb * 64 * 16 * 4 + 4 * 5120 * 18 * 4
    assert one < max(old_one, ch_one) + 4096
    assert lib.ss_bwd_workspace_size(0, 1, 16, 1) == ctypes.c_size_t(-1).value


def test_bwd_path_rejects_invalid_arguments(lib):
    """Argument checks run before any device query."""
    assert lib.ss_bwd_path(0, 1, 16, 1, 1, None) == -1
    assert lib.ss_bwd_path(1, 1, 8, 1, 1, None) == -1      # dstate must be 16
    assert lib.ss_bwd_path(1, 1, 16, 1, 7, None) == -1     # unknown dtype
    assert b"dtype" in lib.ss_last_error()


def test_binding_refuses_cpu_tensors(lib):
    import torch
    u = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError, match="CUDA"):
        ops.ss_fwd(u, u, torch.zeros(2, 16), torch.zeros(1, 16, 8), torch.zeros(1, 16, 8))


def test_ssd_bwd_workspace_and_argument_checks(lib):
    """The SSD backward's workspace holds the chunk maps of the state and the
    adjoint (b, nh, chunks, 64, N) twice, the per-head dB/dC (b, L, nh, N) twice
    and four per-chunk arrays; bad shapes are refused before any launch."""
    n = lib.ss_ssd_bwd_workspace_size(4, 4096, 80, 64, 1, 128)
    maps = 2 * 4 * 80 * 64 * 64 * 128 * 4
    per_head = 2 * 4 * 4096 * 80 * 128 * 4
    per_chunk = 4 * (4 * 80 * 64 * 4)
    assert maps + per_head + per_chunk <= n <= maps + per_head + per_chunk + 8 * 256
    bad = ctypes.c_size_t(-1).value
    assert lib.ss_ssd_bwd_workspace_size(1, 16, 3, 64, 2, 64) == bad     # ngroups must divide nheads
    assert lib.ss_ssd_bwd_workspace_size(1, 16, 2, 32, 1, 64) == bad     # headdim 64 only
    assert lib.ss_ssd_bwd_workspace_size(1, 16, 2, 64, 1, 96) == bad     # dstate 64 or 128
    P = ctypes.c_void_p
    args = [P(256)] * 5 + [None] * 3 + [1, None, P(256), None] + [P(256)] * 5 + [None] * 4 + [P(256), 1 << 30, None]
    assert lib.ss_ssd_bwd(1, 16, 2, 64, 1, 64, 0, *args) == 2            # fp32 storage: unsupported
    assert lib.ss_ssd_bwd(0, 16, 2, 64, 1, 64, 1, *args) == 1            # empty batch
    assert b"positive" in lib.ss_last_error()
    no_dy = list(args)
    no_dy[10] = None
    assert lib.ss_ssd_bwd(1, 16, 2, 64, 1, 64, 1, *no_dy) == 1           # dy is required


def test_sequence_sharding_and_path_entry_points_validate_on_the_host(lib, monkeypatch):
    """ss_segment_decay and ss_state_chain refuse bad arguments before any
    launch; ss_ssd_fwd_path reads SS_SSD_VARIANT."""
    P = lambda v: None if v is None else ctypes.c_void_p(v)

    def decay(batch=2, dim=4, dstate=16, seqlen=8, dtype=1, delta=16, A=16, P_out=16):
        return lib.ss_segment_decay(batch, dim, dstate, seqlen, dtype, P(delta), P(A), None, 1, P(P_out), None)

    assert decay(batch=0) == 1 and b"positive" in lib.ss_last_error()
    assert decay(dstate=300) == 2
    assert decay(dtype=7) == 2
    assert decay(delta=None) == 1
    assert decay(delta=17) == 3                    # bf16 data not 2-byte aligned
    assert decay(A=18) == 3                        # fp32 not 4-byte aligned

    def chain(count=64, nseg=3, p=16, e=16, init=None, out=16):
        return lib.ss_state_chain(count, nseg, P(p), P(e), P(init), 0, P(out), None)

    assert chain(count=0) == 1
    assert chain(nseg=70000) == 2
    assert chain(count=1 << 39) == 2
    assert chain(p=None) == 1
    assert chain(out=None) == 1
    assert chain(init=6) == 3

    monkeypatch.delenv("SS_SSD_VARIANT", raising=False)
    assert lib.ss_ssd_fwd_path() == 0              # SS_SSD_PATH_TCGEN05
    monkeypatch.setenv("SS_SSD_VARIANT", "mma")
    assert lib.ss_ssd_fwd_path() == 1              # SS_SSD_PATH_MMA
