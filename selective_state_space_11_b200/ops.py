"""Python binding of libss.so (include/ss.h): argument marshalling only.

Every step of the scan runs in the library's CUDA kernels; this module checks
tensors, allocates outputs and workspace with PyTorch (device memory is the
only thing PyTorch provides), passes raw pointers and the current stream, and
turns a non-OK status into an exception.  There is no CPU or PyTorch fallback:
if libss.so is missing or a tensor is not on a CUDA device, calls raise.

Names follow the C ABI: ss_fwd, ss_bwd, ss_state_update; selective_scan_fn
wraps ss_fwd/ss_bwd as a torch.autograd.Function with the argument list of
"Mamba" (stanleyjacob.dev), Part IV Stage 5 (selective_scan_fn).
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Tuple

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libss.so")
CHUNK = 64
DSTATE = 16

SS_F32, SS_BF16, SS_F16 = 0, 1, 2
_DTYPE = {torch.float32: SS_F32, torch.bfloat16: SS_BF16, torch.float16: SS_F16}
STATUS = {0: "SS_OK", 1: "SS_ERR_INVALID_ARG", 2: "SS_ERR_UNSUPPORTED", 3: "SS_ERR_ALIGNMENT",
          4: "SS_ERR_WORKSPACE", 5: "SS_ERR_CUDA", 6: "SS_ERR_INTERNAL"}

# Every symbol include/ss.h declares, with its ctypes signature.
_P, _I64, _I, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "ss_version": ([], _I),
    "ss_last_error": ([], ctypes.c_char_p),
    "ss_status_string": ([_I], ctypes.c_char_p),
    "ss_fwd_path": ([_I64, _I64, _I64, _I64, ctypes.POINTER(ctypes.c_int64)], _I),
    "ss_fwd_workspace_size": ([_I64, _I64, _I64, _I64], _SZ),
    "ss_fwd": ([_I64, _I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P,
                _P, _SZ, _P], _I),
    "ss_fwd_with_state": ([_I64, _I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P,
                           _P, _P, _P, _P, _SZ, _P], _I),
    "ss_fwd_noalloc": ([_I64, _I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P,
                        _P, _P], _I),
    "ss_bwd_workspace_size": ([_I64, _I64, _I64, _I64], _SZ),
    "ss_bwd_path": ([_I64, _I64, _I64, _I64, _I, ctypes.POINTER(ctypes.c_int64)], _I),
    "ss_bwd": ([_I64, _I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P,
                _P, _P, _P, _P, _P, _P, _P, _SZ, _P], _I),
    "ss_bwd_with_state": ([_I64, _I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P,
                           _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], _I),
    "ss_conv1d_fwd": ([_I64, _I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _I, _P, _P, _P], _I),
    "ss_conv1d_bwd_workspace_size": ([_I64, _I64, _I64, _I64], _SZ),
    "ss_conv1d_bwd": ([_I64, _I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P,
                       _P, _SZ, _P], _I),
    "ss_conv1d_step": ([_I64, _I64, _I64, _I, _P, _P, _P, _P, _I, _P, _P], _I),
    "ss_ssd_fwd": ([_I64, _I64, _I64, _I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P,
                    _P, _P, _P], _I),
    "ss_segment_decay": ([_I64, _I64, _I64, _I64, _I, _P, _P, _P, _I, _P, _P], _I),
    "ss_state_chain": ([_I64, _I64, _P, _P, _P, _I, _P, _P], _I),
    "ss_ssd_fwd_path": ([], _I),
    "ss_device_fault": ([_I], _I),
    "ss_ssd_bwd_workspace_size": ([_I64, _I64, _I64, _I64, _I64, _I64], _SZ),
    "ss_ssd_bwd": ([_I64, _I64, _I64, _I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P,
                    _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], _I),
    "ss_state_update": ([_I64, _I64, _I64, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P],
                        _I),
}

_lib = None


class SSError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libss.so (built in-tree by __graft_entry__.build / build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m selective_state_space_11_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(l, name)
            fn.argtypes = args
            fn.restype = res
        _lib = l
    return _lib


def _check(status: int):
    if status != 0:
        raise SSError(status, lib().ss_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _need(t: Optional[torch.Tensor], name: str, shape, dtype, dev, optional=False):
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if t.device != dev:
        raise ValueError(f"{name} is on {t.device}, expected {dev}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_inputs(u, delta, A, B, C, D, z, delta_bias):
    if u.dtype not in _DTYPE:
        raise ValueError(f"unsupported dtype {u.dtype}")
    bsz, dim, L = u.shape
    N = A.shape[-1]
    dev = u.device
    _need(u, "u", (bsz, dim, L), u.dtype, dev)
    _need(delta, "delta", (bsz, dim, L), u.dtype, dev)
    _need(z, "z", (bsz, dim, L), u.dtype, dev, optional=True)
    _need(A, "A", (dim, N), torch.float32, dev)
    _need(B, "B", (bsz, N, L), u.dtype, dev)
    _need(C, "C", (bsz, N, L), u.dtype, dev)
    _need(D, "D", (dim,), torch.float32, dev, optional=True)
    _need(delta_bias, "delta_bias", (dim,), torch.float32, dev, optional=True)
    return bsz, dim, N, L, dev


def fwd_path(batch: int, dim: int, seqlen: int, dstate: int = DSTATE) -> Tuple[int, int]:
    """(path, num_segments) the library picks on the current device."""
    nseg = ctypes.c_int64(0)
    path = lib().ss_fwd_path(batch, dim, dstate, seqlen, ctypes.byref(nseg))
    if path < 0:
        raise SSError(1, lib().ss_last_error().decode())
    return path, nseg.value


def bwd_path(batch: int, dim: int, seqlen: int, dtype: str = "bf16",
             dstate: int = DSTATE) -> Tuple[int, int]:
    """(walk variant, chunk groups) the backward picks on the current device."""
    ng = ctypes.c_int64(0)
    code = {"f32": SS_F32, "bf16": SS_BF16, "f16": SS_F16}[dtype]
    v = lib().ss_bwd_path(batch, dim, dstate, seqlen, code, ctypes.byref(ng))
    if v < 0:
        raise SSError(1, lib().ss_last_error().decode())
    return v, ng.value


def ss_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
           final_state=True, checkpoints=True, out=None, workspace=None, h0=None, seq_idx=None):
    """Forward scan.  Returns (y, final_state or None, checkpoints or None).

    u, delta, z: (batch, dim, L) in bf16/fp16/fp32; A: (dim, 16) fp32;
    B, C: (batch, 16, L); D, delta_bias: (dim,) fp32; h0: (batch, dim, 16) fp32
    initial state or None (zero); seq_idx: (batch, L) int32 packed-document ids
    (the state restarts wherever the id changes) or None.  ``out`` may supply preallocated
    (y, final_state, checkpoints); ``workspace`` a uint8 tensor.
    """
    bsz, dim, N, L, dev = _check_inputs(u, delta, A, B, C, D, z, delta_bias)
    _need(h0, "h0", (bsz, dim, N), torch.float32, dev, optional=True)
    _need(seq_idx, "seq_idx", (bsz, L), torch.int32, dev, optional=True)
    nck = (L + CHUNK - 1) // CHUNK
    if out is not None:
        y, fs, ck = out
        _need(y, "y", (bsz, dim, L), u.dtype, dev)
        _need(fs, "final_state", (bsz, dim, N), torch.float32, dev, optional=True)
        _need(ck, "checkpoints", (bsz, dim, nck, N), torch.float32, dev, optional=True)
    else:
        y = torch.empty_like(u)
        fs = torch.empty(bsz, dim, N, device=dev, dtype=torch.float32) if final_state else None
        ck = torch.empty(bsz, dim, nck, N, device=dev, dtype=torch.float32) if checkpoints else None
    with torch.cuda.device(dev):
        need = lib().ss_fwd_workspace_size(bsz, dim, N, L)
        if need == ctypes.c_size_t(-1).value:
            _check(1)
        if need and (workspace is None or workspace.numel() < need):
            workspace = torch.empty(need, device=dev, dtype=torch.uint8)
        _check(lib().ss_fwd_with_state(bsz, dim, N, L, _DTYPE[u.dtype], _ptr(u), _ptr(delta),
                                       _ptr(z), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                       _ptr(delta_bias), int(bool(delta_softplus)), _ptr(h0),
                                       _ptr(seq_idx), _ptr(y), _ptr(fs), _ptr(ck),
                                       _ptr(workspace) if need else None, need, _stream(dev)))
    return y, fs, ck


def ss_fwd_noalloc(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
                   out=None):
    """ss_fwd without a workspace argument: the library's built-in scratch area
    is used (for hosts that must not allocate device memory at call time).

    ``out`` = (y, final_state or None, checkpoints or None), preallocated by the
    caller; returns it.  Raises SSError(SS_ERR_WORKSPACE) for problems whose
    scratch need exceeds the built-in area.
    """
    bsz, dim, N, L, dev = _check_inputs(u, delta, A, B, C, D, z, delta_bias)
    y, fs, ck = out
    _need(y, "y", (bsz, dim, L), u.dtype, dev)
    _need(fs, "final_state", (bsz, dim, N), torch.float32, dev, optional=True)
    _need(ck, "checkpoints", (bsz, dim, (L + CHUNK - 1) // CHUNK, N), torch.float32, dev,
          optional=True)
    with torch.cuda.device(dev):
        _check(lib().ss_fwd_noalloc(bsz, dim, N, L, _DTYPE[u.dtype], _ptr(u), _ptr(delta), _ptr(z),
                                    _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(delta_bias),
                                    int(bool(delta_softplus)), _ptr(y), _ptr(fs), _ptr(ck),
                                    _stream(dev)))
    return y, fs, ck


def ss_bwd(u, delta, A, B, C, dy, checkpoints, D=None, z=None, delta_bias=None,
           delta_softplus=True, workspace=None, out=None, h0=None, dfinal=None,
           want_dh0=None, seq_idx=None) -> Dict[str, Optional[torch.Tensor]]:
    """Backward scan for the loss <dy, y> + <dfinal, final_state>; ``checkpoints``
    come from ss_fwd on the same inputs (and the same h0).

    Returns du, ddelta, dz (input dtype), dA, dB, dC, dD, ddelta_bias and dh0
    (fp32; dh0 only when ``want_dh0``, which defaults to "h0 or dfinal given").
    ``out`` may supply any of these preallocated (same keys).
    """
    bsz, dim, N, L, dev = _check_inputs(u, delta, A, B, C, D, z, delta_bias)
    _need(dy, "dy", (bsz, dim, L), u.dtype, dev)
    _need(h0, "h0", (bsz, dim, N), torch.float32, dev, optional=True)
    _need(dfinal, "dfinal", (bsz, dim, N), torch.float32, dev, optional=True)
    _need(seq_idx, "seq_idx", (bsz, L), torch.int32, dev, optional=True)
    if want_dh0 is None:
        want_dh0 = h0 is not None or dfinal is not None
    _need(checkpoints, "checkpoints", (bsz, dim, (L + CHUNK - 1) // CHUNK, N), torch.float32, dev)
    shapes = dict(du=((bsz, dim, L), u.dtype), ddelta=((bsz, dim, L), u.dtype),
                  dz=((bsz, dim, L), u.dtype), dA=((dim, N), torch.float32),
                  dB=((bsz, N, L), torch.float32), dC=((bsz, N, L), torch.float32),
                  dD=((dim,), torch.float32), ddelta_bias=((dim,), torch.float32),
                  dh0=((bsz, dim, N), torch.float32))
    out = dict(out or {})
    g = {}
    for k, (shp, dt) in shapes.items():
        if (k == "dz" and z is None) or (k == "dh0" and not want_dh0):
            g[k] = None
        elif out.get(k) is not None:
            _need(out[k], k, shp, dt, dev)
            g[k] = out[k]
        else:
            g[k] = torch.empty(shp, device=dev, dtype=dt)
    with torch.cuda.device(dev):
        need = lib().ss_bwd_workspace_size(bsz, dim, N, L)
        if need == ctypes.c_size_t(-1).value:
            _check(1)
        if workspace is None or workspace.numel() < need:
            workspace = torch.empty(need, device=dev, dtype=torch.uint8)
        _check(lib().ss_bwd_with_state(bsz, dim, N, L, _DTYPE[u.dtype], _ptr(u), _ptr(delta),
                                       _ptr(z), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                       _ptr(delta_bias), int(bool(delta_softplus)), _ptr(h0),
                                       _ptr(seq_idx), _ptr(dy), _ptr(dfinal), _ptr(checkpoints),
                                       _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dz"]),
                                       _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dD"]),
                                       _ptr(g["ddelta_bias"]), _ptr(g["dh0"]), _ptr(workspace),
                                       need, _stream(dev)))
    return g


def segment_decay(delta, A, delta_bias=None, delta_softplus=True, out=None):
    """The diagonal state transition of a segment: P = exp(A * sum_t Delta_t),
    (batch, dim, N) fp32, for delta (batch, dim, L)."""
    if delta.dtype not in _DTYPE:
        raise ValueError(f"unsupported dtype {delta.dtype}")
    bsz, dim, L = delta.shape
    N = A.shape[-1]
    dev = delta.device
    _need(delta, "delta", (bsz, dim, L), delta.dtype, dev)
    _need(A, "A", (dim, N), torch.float32, dev)
    _need(delta_bias, "delta_bias", (dim,), torch.float32, dev, optional=True)
    P = out if out is not None else torch.empty(bsz, dim, N, device=dev, dtype=torch.float32)
    _need(P, "P", (bsz, dim, N), torch.float32, dev)
    with torch.cuda.device(dev):
        _check(lib().ss_segment_decay(bsz, dim, N, L, _DTYPE[delta.dtype], _ptr(delta), _ptr(A),
                                      _ptr(delta_bias), int(bool(delta_softplus)), _ptr(P), _stream(dev)))
    return P


def state_chain(P, E, init=None, reverse=False, out=None):
    """Chain segment slabs: P, E (nseg, ...) fp32; returns out (nseg, ...) with
    out[0] = init, out[s+1] = P[s] out[s] + E[s] (reverse: out[-1] = init,
    out[s-1] = P[s] out[s] + E[s]); init (...) fp32 or None (zero)."""
    dev = P.device
    nseg = P.shape[0]
    count = P[0].numel()
    _need(P, "P", tuple(P.shape), torch.float32, dev)
    _need(E, "E", tuple(P.shape), torch.float32, dev)
    _need(init, "init", tuple(P.shape[1:]), torch.float32, dev, optional=True)
    o = out if out is not None else torch.empty_like(P)
    _need(o, "out", tuple(P.shape), torch.float32, dev)
    with torch.cuda.device(dev):
        _check(lib().ss_state_chain(count, nseg, _ptr(P), _ptr(E), _ptr(init), int(bool(reverse)), _ptr(o),
                                    _stream(dev)))
    return o


def ss_state_update(state, u, delta, A, B, C, D=None, z=None, delta_bias=None,
                    delta_softplus=True, y=None):
    """One decode step; ``state`` (batch, dim, 16) fp32 is updated in place.

    u, delta, z: (batch, dim); B, C: (batch, 16).  Returns y (batch, dim).
    """
    if u.dtype not in _DTYPE:
        raise ValueError(f"unsupported dtype {u.dtype}")
    bsz, dim = u.shape
    N = A.shape[-1]
    dev = u.device
    _need(state, "state", (bsz, dim, N), torch.float32, dev)
    _need(u, "u", (bsz, dim), u.dtype, dev)
    _need(delta, "delta", (bsz, dim), u.dtype, dev)
    _need(z, "z", (bsz, dim), u.dtype, dev, optional=True)
    _need(A, "A", (dim, N), torch.float32, dev)
    _need(B, "B", (bsz, N), u.dtype, dev)
    _need(C, "C", (bsz, N), u.dtype, dev)
    _need(D, "D", (dim,), torch.float32, dev, optional=True)
    _need(delta_bias, "delta_bias", (dim,), torch.float32, dev, optional=True)
    if y is None:
        y = torch.empty_like(u)
    with torch.cuda.device(dev):
        _check(lib().ss_state_update(bsz, dim, N, _DTYPE[u.dtype], _ptr(state), _ptr(u),
                                     _ptr(delta), _ptr(z), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                     _ptr(delta_bias), int(bool(delta_softplus)), _ptr(y),
                                     _stream(dev)))
    return y


def _check_conv(x, w, bias, state_in):
    if x.dtype not in _DTYPE:
        raise ValueError(f"unsupported dtype {x.dtype}")
    bsz, dim, L = x.shape
    dev = x.device
    W = w.shape[-1]
    _need(x, "x", (bsz, dim, L), x.dtype, dev)
    _need(w, "w", (dim, W), torch.float32, dev)
    _need(bias, "bias", (dim,), torch.float32, dev, optional=True)
    _need(state_in, "state_in", (bsz, dim, W - 1), torch.float32, dev, optional=True)
    return bsz, dim, L, W, dev


def conv1d_fwd(x, w, bias=None, state_in=None, silu=True, state_out=False, out=None,
               seq_idx=None):
    """Causal depthwise conv1d (+ SiLU) before the scan.  Returns (u, state_out or None).

    x: (batch, dim, L); w: (dim, W) fp32, W <= 4; bias: (dim,) fp32; state_in:
    (batch, dim, W-1) fp32 window before t = 0.  ``state_out`` True (allocate) or a
    tensor receives the last W-1 inputs.  ``out`` may supply u.  seq_idx: (batch, L)
    int32 packed-document ids (the window restarts wherever the id changes) or None.
    """
    bsz, dim, L, W, dev = _check_conv(x, w, bias, state_in)
    _need(seq_idx, "seq_idx", (bsz, L), torch.int32, dev, optional=True)
    u = out if out is not None else torch.empty_like(x)
    _need(u, "u", (bsz, dim, L), x.dtype, dev)
    so = state_out
    if so is True:
        so = torch.empty(bsz, dim, W - 1, device=dev, dtype=torch.float32)
    elif so is False:
        so = None
    _need(so, "state_out", (bsz, dim, W - 1), torch.float32, dev, optional=True)
    with torch.cuda.device(dev):
        _check(lib().ss_conv1d_fwd(bsz, dim, L, W, _DTYPE[x.dtype], _ptr(x), _ptr(w), _ptr(bias),
                                   _ptr(state_in), _ptr(seq_idx), int(bool(silu)), _ptr(u), _ptr(so),
                                   _stream(dev)))
    return u, so


def conv1d_bwd(x, w, du, bias=None, state_in=None, silu=True, dstate_out=None,
               want_dstate_in=None, workspace=None, seq_idx=None) -> Dict[str, Optional[torch.Tensor]]:
    """Adjoint of conv1d_fwd for <du, u> + <dstate_out, state_out>.

    Returns dx (input dtype), dw (dim, W), dbias (dim,) and dstate_in
    (batch, dim, W-1; only when ``want_dstate_in``, default "state_in given").
    """
    bsz, dim, L, W, dev = _check_conv(x, w, bias, state_in)
    _need(du, "du", (bsz, dim, L), x.dtype, dev)
    _need(dstate_out, "dstate_out", (bsz, dim, W - 1), torch.float32, dev, optional=True)
    _need(seq_idx, "seq_idx", (bsz, L), torch.int32, dev, optional=True)
    if want_dstate_in is None:
        want_dstate_in = state_in is not None
    g = dict(dx=torch.empty_like(x), dw=torch.empty(dim, W, device=dev, dtype=torch.float32),
             dbias=torch.empty(dim, device=dev, dtype=torch.float32),
             dstate_in=torch.empty(bsz, dim, W - 1, device=dev, dtype=torch.float32)
             if want_dstate_in else None)
    with torch.cuda.device(dev):
        need = lib().ss_conv1d_bwd_workspace_size(bsz, dim, L, W)
        if need == ctypes.c_size_t(-1).value:
            _check(1)
        if workspace is None or workspace.numel() < need:
            workspace = torch.empty(need, device=dev, dtype=torch.uint8)
        _check(lib().ss_conv1d_bwd(bsz, dim, L, W, _DTYPE[x.dtype], _ptr(x), _ptr(w), _ptr(bias),
                                   _ptr(state_in), _ptr(seq_idx), int(bool(silu)), _ptr(du),
                                   _ptr(dstate_out),
                                   _ptr(g["dx"]), _ptr(g["dw"]), _ptr(g["dbias"]),
                                   _ptr(g["dstate_in"]), _ptr(workspace), need, _stream(dev)))
    return g


def conv1d_step(state, x, w, bias=None, silu=True, u=None):
    """One decode step of the convolution; ``state`` (batch, dim, W-1) fp32 is
    advanced in place.  x: (batch, dim).  Returns u (batch, dim)."""
    if x.dtype not in _DTYPE:
        raise ValueError(f"unsupported dtype {x.dtype}")
    bsz, dim = x.shape
    dev = x.device
    W = w.shape[-1]
    _need(state, "state", (bsz, dim, W - 1), torch.float32, dev)
    _need(w, "w", (dim, W), torch.float32, dev)
    _need(bias, "bias", (dim,), torch.float32, dev, optional=True)
    if u is None:
        u = torch.empty_like(x)
    _need(u, "u", (bsz, dim), x.dtype, dev)
    with torch.cuda.device(dev):
        _check(lib().ss_conv1d_step(bsz, dim, W, _DTYPE[x.dtype], _ptr(state), _ptr(x), _ptr(w),
                                    _ptr(bias), int(bool(silu)), _ptr(u), _stream(dev)))
    return u


class _CausalConv1d(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, w, bias, silu):
        u, _ = conv1d_fwd(x, w, bias=bias, silu=silu)
        ctx.save_for_backward(x, w, bias)
        ctx.silu = silu
        return u

    @staticmethod
    def backward(ctx, du):
        x, w, bias = ctx.saved_tensors
        g = conv1d_bwd(x, w, du.contiguous(), bias=bias, silu=ctx.silu)
        return g["dx"], g["dw"], g["dbias"] if bias is not None else None, None


def causal_conv1d_fn(x, w, bias=None, silu=True):
    """Differentiable causal depthwise conv1d (+ SiLU): x (batch, dim, L), w (dim, W)."""
    return _CausalConv1d.apply(x, w, bias, silu)


def ssd_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True, h0=None,
            final_state=True, out=None):
    """Mamba-2 SSD forward.  Returns (y, final_state or None).

    x, z: (batch, L, nheads, 64) bf16/fp16; dt: (batch, L, nheads); A, D, dt_bias:
    (nheads,) fp32; B, C: (batch, L, ngroups, dstate), dstate 64 or 128; h0:
    (batch, nheads, 64, dstate) fp32.  ``out`` may supply y.
    """
    if x.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError(f"unsupported dtype {x.dtype} (bf16 or fp16)")
    bsz, L, nh, P = x.shape
    ng, N = B.shape[2], B.shape[3]
    dev = x.device
    _need(x, "x", (bsz, L, nh, P), x.dtype, dev)
    _need(dt, "dt", (bsz, L, nh), x.dtype, dev)
    _need(A, "A", (nh,), torch.float32, dev)
    _need(B, "B", (bsz, L, ng, N), x.dtype, dev)
    _need(C, "C", (bsz, L, ng, N), x.dtype, dev)
    _need(D, "D", (nh,), torch.float32, dev, optional=True)
    _need(z, "z", (bsz, L, nh, P), x.dtype, dev, optional=True)
    _need(dt_bias, "dt_bias", (nh,), torch.float32, dev, optional=True)
    _need(h0, "h0", (bsz, nh, P, N), torch.float32, dev, optional=True)
    y = out if out is not None else torch.empty_like(x)
    _need(y, "y", (bsz, L, nh, P), x.dtype, dev)
    fs = torch.empty(bsz, nh, P, N, device=dev, dtype=torch.float32) if final_state is True else \
        (final_state if final_state is not False else None)
    _need(fs, "final_state", (bsz, nh, P, N), torch.float32, dev, optional=True)
    with torch.cuda.device(dev):
        _check(lib().ss_ssd_fwd(bsz, L, nh, P, ng, N, _DTYPE[x.dtype], _ptr(x), _ptr(dt), _ptr(A),
                                _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
                                int(bool(dt_softplus)), _ptr(h0), _ptr(y), _ptr(fs), _stream(dev)))
    return y, fs


def ssd_bwd(x, dt, A, B, C, dy, D=None, z=None, dt_bias=None, dt_softplus=True, h0=None,
            dfinal=None, workspace=None):
    """Mamba-2 SSD backward: the gradient of <dy, y> + <dfinal, final_state> of
    ``ssd_fwd`` with respect to its inputs.  Returns a dict with dx, ddt, dz (None
    without z) in the input dtype; dB, dC (batch, L, ngroups, dstate), dA, dD,
    ddt_bias (nheads,) and dh0 (batch, nheads, 64, dstate) in fp32.  ``workspace``
    (uint8, at least ``ss_ssd_bwd_workspace_size`` bytes) is allocated when absent.
    """
    if x.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError(f"unsupported dtype {x.dtype} (bf16 or fp16)")
    bsz, L, nh, P = x.shape
    ng, N = B.shape[2], B.shape[3]
    dev = x.device
    _need(x, "x", (bsz, L, nh, P), x.dtype, dev)
    _need(dt, "dt", (bsz, L, nh), x.dtype, dev)
    _need(A, "A", (nh,), torch.float32, dev)
    _need(B, "B", (bsz, L, ng, N), x.dtype, dev)
    _need(C, "C", (bsz, L, ng, N), x.dtype, dev)
    _need(dy, "dy", (bsz, L, nh, P), x.dtype, dev)
    _need(D, "D", (nh,), torch.float32, dev, optional=True)
    _need(z, "z", (bsz, L, nh, P), x.dtype, dev, optional=True)
    _need(dt_bias, "dt_bias", (nh,), torch.float32, dev, optional=True)
    _need(h0, "h0", (bsz, nh, P, N), torch.float32, dev, optional=True)
    _need(dfinal, "dfinal", (bsz, nh, P, N), torch.float32, dev, optional=True)
    f32 = dict(device=dev, dtype=torch.float32)
    g = dict(dx=torch.empty_like(x), ddt=torch.empty_like(dt),
             dz=torch.empty_like(z) if z is not None else None,
             dB=torch.empty(bsz, L, ng, N, **f32), dC=torch.empty(bsz, L, ng, N, **f32),
             dA=torch.empty(nh, **f32), dD=torch.empty(nh, **f32), ddt_bias=torch.empty(nh, **f32),
             dh0=torch.empty(bsz, nh, P, N, **f32))
    with torch.cuda.device(dev):
        need = lib().ss_ssd_bwd_workspace_size(bsz, L, nh, P, ng, N)
        if need == ctypes.c_size_t(-1).value:
            _check(2)
        if workspace is None or workspace.numel() < need:
            workspace = torch.empty(need, device=dev, dtype=torch.uint8)
        _check(lib().ss_ssd_bwd(bsz, L, nh, P, ng, N, _DTYPE[x.dtype], _ptr(x), _ptr(dt), _ptr(A),
                                _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
                                int(bool(dt_softplus)), _ptr(h0), _ptr(dy), _ptr(dfinal),
                                _ptr(g["dx"]), _ptr(g["ddt"]), _ptr(g["dA"]), _ptr(g["dB"]),
                                _ptr(g["dC"]), _ptr(g["dD"]), _ptr(g["dz"]), _ptr(g["ddt_bias"]),
                                _ptr(g["dh0"]), _ptr(workspace), int(workspace.numel()), _stream(dev)))
    return g


class _SelectiveScan(torch.autograd.Function):
    @staticmethod
    def forward(ctx, u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, return_last_state):
        y, last, ck = ss_fwd(u, delta, A, B, C, D=D, z=z, delta_bias=delta_bias,
                             delta_softplus=delta_softplus, final_state=return_last_state,
                             checkpoints=True, h0=h0)
        ctx.save_for_backward(u, delta, A, B, C, D, z, delta_bias, ck, h0)
        ctx.softplus = delta_softplus
        return (y, last) if return_last_state else y

    @staticmethod
    def backward(ctx, dy, dlast=None):
        u, delta, A, B, C, D, z, delta_bias, ck, h0 = ctx.saved_tensors
        g = ss_bwd(u, delta, A, B, C, dy.contiguous(), ck, D=D, z=z, delta_bias=delta_bias,
                   delta_softplus=ctx.softplus, h0=h0,
                   dfinal=dlast.contiguous() if dlast is not None else None,
                   want_dh0=h0 is not None)
        return (g["du"], g["ddelta"], g["dA"], g["dB"].to(B.dtype), g["dC"].to(C.dtype),
                g["dD"] if D is not None else None, g["dz"],
                g["ddelta_bias"] if delta_bias is not None else None, None, g["dh0"], None)


class _SSD(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, dt, A, B, C, D, z, dt_bias, dt_softplus, h0, return_final_state):
        y, fs = ssd_fwd(x, dt, A, B, C, D=D, z=z, dt_bias=dt_bias, dt_softplus=dt_softplus, h0=h0,
                        final_state=bool(return_final_state))
        ctx.save_for_backward(x, dt, A, B, C, D, z, dt_bias, h0)
        ctx.softplus = dt_softplus
        return (y, fs) if return_final_state else y

    @staticmethod
    def backward(ctx, dy, dfs=None):
        x, dt, A, B, C, D, z, dt_bias, h0 = ctx.saved_tensors
        g = ssd_bwd(x, dt, A, B, C, dy.contiguous(), D=D, z=z, dt_bias=dt_bias,
                    dt_softplus=ctx.softplus, h0=h0,
                    dfinal=dfs.contiguous() if dfs is not None else None)
        return (g["dx"], g["ddt"], g["dA"], g["dB"].to(B.dtype), g["dC"].to(C.dtype),
                g["dD"] if D is not None else None, g["dz"],
                g["ddt_bias"] if dt_bias is not None else None, None,
                g["dh0"] if h0 is not None else None, None)


def ssd_fn(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True, h0=None,
           return_final_state=False):
    """Differentiable Mamba-2 SSD: ``ssd_fwd`` forward, ``ssd_bwd`` backward.

    x, z: (batch, L, nheads, 64); dt: (batch, L, nheads); B, C: (batch, L, ngroups,
    dstate) in bf16/fp16; A, D, dt_bias: (nheads,) fp32; h0: (batch, nheads, 64,
    dstate) fp32 or None (gradient flows into it).  return_final_state: also return
    the final state (its gradient flows back).
    """
    return _SSD.apply(x, dt, A, B, C, D, z, dt_bias, dt_softplus, h0, return_final_state)


def selective_scan_fn(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=False,
                      h0=None, return_last_state=False):
    """Differentiable scan: y = (C.h + D u) SiLU(z) with checkpointed backward.

    h0: (batch, dim, 16) fp32 initial state (gradient flows into it) or None.
    return_last_state: also return the final state (its gradient flows back).
    """
    return _SelectiveScan.apply(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0,
                                return_last_state)
