"""Seeded synthetic inputs for the selective scan -- shared by tests and bench.

This module holds the input recipe only: random draws, dtype rounding and the
named layer shapes.  It contains none of the scan's arithmetic, and both the
fp64 oracle and the CUDA path are fed from it, so the two see identical bits.

Recipe (the pages use Mamba layer shapes, no dataset):
  u, delta, z ~ N(0, 1)           shape (batch, dim, L)
  B, C        ~ N(0, 1)           shape (batch, N, L), shared across channels
  delta_bias  = log(expm1(v)), v ~ U(1e-3, 0.1)  (the softplus preimage of v)
  A           = -exp(A_log), A_log[d, n] = log(n + 1)  so A[d, n] = -(n + 1)
  D           ~ U(0, 1)
  dy          ~ N(0, 1)           upstream gradient for the backward
Values are drawn in fp32 and, for a bf16 workload, rounded once (RNE) to bf16.
A, D and delta_bias stay fp32.  Shapes follow "Mamba" (stanleyjacob.dev),
Part IV Stage 5 (selective_scan_fn) and Part VII Lab 5 (d_inner = 1536 for
d_model 768); the B=1, D=16, L=32768 shape is the microbenchmark of the
"mamba-metal" README, section "Status".
"""
from __future__ import annotations

import dataclasses

from typing import Dict, Optional

import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    dim: int
    dstate: int
    seqlen: int
    dtype: str          # "f32", "bf16" or "f16": storage type of u, delta, z, B, C, y, grads
    seed: int
    decode_steps: int = 0


# The five named workloads: a tiny parity case, the pages' microbenchmark
# shape, two Mamba layer shapes and a long-context prefill followed by decode.
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 2, 64, 16, 200, "f32", 1000),
    "microbench": Workload("microbench", 1, 16, 16, 32768, "f32", 1001),
    "mamba130m_layer": Workload("mamba130m_layer", 8, 1536, 16, 2048, "bf16", 1002),
    "mamba2.8b_layer": Workload("mamba2.8b_layer", 4, 5120, 16, 4096, "bf16", 1003),
    "long_prefill_decode": Workload("long_prefill_decode", 1, 2048, 16, 65536, "bf16", 1004,
                                    decode_steps=256),
}

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_inputs(batch: int, dim: int, dstate: int, seqlen: int, dtype: str = "f32",
                seed: int = 0, device="cpu", with_z: bool = True, with_D: bool = True,
                with_bias: bool = True, with_dy: bool = True) -> Dict[str, Optional[torch.Tensor]]:
    """Draw one scan problem.  Data tensors are in ``dtype``; A, D, delta_bias fp32."""
    dev = torch.device(device)
    g = _gen(seed, dev)
    tdt = TORCH_DTYPE[dtype]

    def normal(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32).to(tdt)

    out: Dict[str, Optional[torch.Tensor]] = {}
    out["u"] = normal(batch, dim, seqlen)
    out["delta"] = normal(batch, dim, seqlen)
    out["z"] = normal(batch, dim, seqlen) if with_z else None
    out["B"] = normal(batch, dstate, seqlen)
    out["C"] = normal(batch, dstate, seqlen)
    a_log = torch.log(torch.arange(1, dstate + 1, device=dev, dtype=torch.float32))
    out["A"] = (-torch.exp(a_log)).unsqueeze(0).repeat(dim, 1).contiguous()
    if with_D:
        out["D"] = torch.rand(dim, generator=g, device=dev, dtype=torch.float32)
    else:
        out["D"] = None
    if with_bias:
        v = torch.rand(dim, generator=g, device=dev, dtype=torch.float64) * (0.1 - 1e-3) + 1e-3
        out["delta_bias"] = torch.log(torch.expm1(v)).to(torch.float32)
    else:
        out["delta_bias"] = None
    out["dy"] = normal(batch, dim, seqlen) if with_dy else None
    return out


def make_decode_tokens(batch: int, dim: int, dstate: int, steps: int, dtype: str = "f32",
                       seed: int = 0, device="cpu") -> Dict[str, torch.Tensor]:
    """Fresh N(0,1) per-token inputs for ``steps`` decode steps.

    u, delta, z: (steps, batch, dim); B, C: (steps, batch, N).
    """
    dev = torch.device(device)
    g = _gen(seed + 7919, dev)
    tdt = TORCH_DTYPE[dtype]

    def normal(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32).to(tdt)

    return dict(u=normal(steps, batch, dim), delta=normal(steps, batch, dim),
                z=normal(steps, batch, dim), B=normal(steps, batch, dstate),
                C=normal(steps, batch, dstate))


def make_conv_inputs(batch: int, dim: int, seqlen: int, width: int = 4, dtype: str = "f32",
                     seed: int = 0, device="cpu") -> Dict[str, torch.Tensor]:
    """Inputs of the causal depthwise conv1d that feeds the scan: x ~ N(0,1)
    (batch, dim, L) in the storage dtype; taps w ~ N(0, 1/width) and bias
    ~ N(0, 0.1^2), fp32; an incoming window state ~ N(0,1) (batch, dim, width-1)
    rounded through the storage dtype (it holds earlier inputs); and du ~ N(0,1)."""
    dev = torch.device(device)
    g = _gen(seed + 15485863, dev)
    tdt = TORCH_DTYPE[dtype]

    def normal(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32)

    return dict(x=normal(batch, dim, seqlen).to(tdt),
                w=normal(dim, width) / width ** 0.5,
                bias=normal(dim) * 0.1,
                state=normal(batch, dim, width - 1).to(tdt).float(),
                du=normal(batch, dim, seqlen).to(tdt))


def make_ssd_inputs(batch: int, seqlen: int, nheads: int, headdim: int, ngroups: int, dstate: int,
                    dtype: str = "bf16", seed: int = 0, device="cpu", with_z=True, with_D=True,
                    with_bias=True) -> Dict[str, Optional[torch.Tensor]]:
    """Inputs of the Mamba-2 SSD layer (time-major): x, z ~ N(0,1) (batch, L, nheads,
    headdim); dt ~ N(0,1) (batch, L, nheads); B, C ~ N(0,1) / sqrt(dstate) (batch,
    L, ngroups, dstate), all in the storage dtype; A = -exp(U(0, log 16)) per head
    (Mamba-2's A range 1..16), D ~ U(0,1), dt_bias = log(expm1(U(1e-3, 0.1))), fp32."""
    dev = torch.device(device)
    g = _gen(seed + 32452843, dev)
    tdt = TORCH_DTYPE[dtype]

    def normal(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32)

    def uniform(n, lo, hi):
        return lo + (hi - lo) * torch.rand(n, generator=g, device=dev, dtype=torch.float32)

    x = normal(batch, seqlen, nheads, headdim).to(tdt)
    dt = normal(batch, seqlen, nheads).to(tdt)
    B = (normal(batch, seqlen, ngroups, dstate) / dstate ** 0.5).to(tdt)
    C = (normal(batch, seqlen, ngroups, dstate) / dstate ** 0.5).to(tdt)
    A = -torch.exp(uniform(nheads, 0.0, math.log(16.0)))
    D = uniform(nheads, 0.0, 1.0) if with_D else None
    z = normal(batch, seqlen, nheads, headdim).to(tdt) if with_z else None
    bias = torch.log(torch.expm1(uniform(nheads, 1e-3, 0.1))) if with_bias else None
    return dict(x=x, dt=dt, A=A, B=B, C=C, D=D, z=z, dt_bias=bias)


def make_state(batch: int, dim: int, dstate: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """An N(0,1) fp32 state-shaped tensor (batch, dim, N): an initial state h0
    or a gradient arriving at the final state."""
    dev = torch.device(device)
    g = _gen(seed + 104729, dev)
    return torch.randn(batch, dim, dstate, generator=g, device=dev, dtype=torch.float32)


def workload_inputs(name: str, device="cpu", **kw) -> Dict[str, Optional[torch.Tensor]]:
    w = WORKLOADS[name]
    return make_inputs(w.batch, w.dim, w.dstate, w.seqlen, w.dtype, w.seed, device=device, **kw)


def as_f64(t: Optional[torch.Tensor]):
    """Exact upcast of a stored tensor to a float64 numpy array (None passes through)."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()


