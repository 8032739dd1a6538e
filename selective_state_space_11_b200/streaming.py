"""Scan steps on host-resident batches, with the PCIe copies overlapped.

A training step of the scan on data that lives in (pinned) host memory moves
its inputs u, delta, z, dy, B, C to the device, runs ss_fwd and ss_bwd, and
moves y and every gradient back.  Done one after another, the two copies
(about 670 MB each way at the mamba-2.8b layer shape) take ten times longer
than the kernels.  `HostStepPipeline` keeps two device slots and three CUDA
streams, so that step k+1's inputs are copied in while step k's kernels run
and step k-1's results are copied out: each PCIe direction then runs on its
own copy engine, and the step rate is bound by the slower copy instead of by
their sum.

Per slot, CUDA events order copy-in -> kernels -> copy-out; a slot's inputs
are not overwritten before the kernels that read them have finished, and its
outputs not before they have been copied out.  Every kernel is the library's
own (ss_fwd, ss_bwd through the C ABI); the only other device work is the
copies.
"""
from __future__ import annotations

from typing import Dict

import torch

from . import ops

INPUTS = ("u", "delta", "z", "dy", "B", "C")


class HostStepPipeline:
    """fwd + bwd steps of one problem shape on host batches, copies overlapped.

    ``params`` holds the device-resident parameters A, D, delta_bias (fp32).
    ``step(host_in, host_out)`` enqueues one step: ``host_in`` maps u, delta,
    z, dy, B, C to pinned host tensors of the problem's shapes; ``host_out``
    maps y, du, ddelta, dz, dB, dC, dA, dD, ddelta_bias to pinned host tensors
    that receive the results.  The copies are asynchronous: a step's host
    inputs must keep their contents until its copy-in has run, and its host
    outputs hold the results only after ``synchronize()``.  Copy-outs run in
    step order on one stream, so steps may share output buffers when only the
    last step's results are wanted.  ``allreduce`` (optional) is called on the
    packed parameter gradients after each backward, on the compute stream.
    """

    def __init__(self, batch: int, dim: int, seqlen: int, dtype: torch.dtype, params: Dict,
                 device, dstate: int = ops.DSTATE, with_z: bool = True, allreduce=None):
        self.dev = torch.device(device)
        self.params = params
        self.with_z = with_z
        self.allreduce = allreduce
        nck = (seqlen + ops.CHUNK - 1) // ops.CHUNK
        shp = (batch, dim, seqlen)
        self.slots = []
        for _ in range(2):
            s = {k: torch.empty(shp, device=self.dev, dtype=dtype) for k in ("u", "delta", "dy")}
            s["z"] = torch.empty(shp, device=self.dev, dtype=dtype) if with_z else None
            s["B"] = torch.empty(batch, dstate, seqlen, device=self.dev, dtype=dtype)
            s["C"] = torch.empty(batch, dstate, seqlen, device=self.dev, dtype=dtype)
            s["y"] = torch.empty(shp, device=self.dev, dtype=dtype)
            pg = torch.empty(dim * dstate + 2 * dim, device=self.dev, dtype=torch.float32)
            s["pgrad"] = pg
            s["g"] = dict(du=torch.empty(shp, device=self.dev, dtype=dtype),
                          ddelta=torch.empty(shp, device=self.dev, dtype=dtype),
                          dz=torch.empty(shp, device=self.dev, dtype=dtype) if with_z else None,
                          dB=torch.empty(batch, dstate, seqlen, device=self.dev, dtype=torch.float32),
                          dC=torch.empty(batch, dstate, seqlen, device=self.dev, dtype=torch.float32),
                          dA=pg[:dim * dstate].view(dim, dstate),
                          dD=pg[dim * dstate:dim * dstate + dim],
                          ddelta_bias=pg[dim * dstate + dim:])
            self.slots.append(s)
        # the kernels run one step at a time on the compute stream, so the
        # checkpoints and workspaces can be shared by the two slots
        self.ck = torch.empty(batch, dim, nck, dstate, device=self.dev, dtype=torch.float32)
        with torch.cuda.device(self.dev):
            nf = ops.lib().ss_fwd_workspace_size(batch, dim, dstate, seqlen)
            nb = ops.lib().ss_bwd_workspace_size(batch, dim, dstate, seqlen)
        self.fws = torch.empty(max(int(nf), 16), device=self.dev, dtype=torch.uint8)
        self.bws = torch.empty(int(nb), device=self.dev, dtype=torch.uint8)
        self.s_in = torch.cuda.Stream(self.dev)
        self.s_comp = torch.cuda.Stream(self.dev)
        self.s_out = torch.cuda.Stream(self.dev)
        self.in_done = [torch.cuda.Event() for _ in range(2)]
        self.comp_done = [None, None]
        self.out_done = [None, None]
        self.k = 0

    def step(self, host_in: Dict[str, torch.Tensor], host_out: Dict[str, torch.Tensor]) -> None:
        slot = self.k % 2
        s = self.slots[slot]
        p = self.params
        # ---- copy-in: the slot's inputs are free once the kernels of two steps ago finished
        with torch.cuda.stream(self.s_in):
            if self.comp_done[slot] is not None:
                self.s_in.wait_event(self.comp_done[slot])
            for k in INPUTS:
                if s[k] is not None:
                    s[k].copy_(host_in[k], non_blocking=True)
            self.in_done[slot].record(self.s_in)
        # ---- kernels: wait for this slot's inputs and for its previous outputs to have left
        with torch.cuda.stream(self.s_comp):
            self.s_comp.wait_event(self.in_done[slot])
            if self.out_done[slot] is not None:
                self.s_comp.wait_event(self.out_done[slot])
            ops.ss_fwd(s["u"], s["delta"], p["A"], s["B"], s["C"], D=p.get("D"), z=s["z"],
                       delta_bias=p.get("delta_bias"), delta_softplus=True,
                       out=(s["y"], None, self.ck), workspace=self.fws)
            ops.ss_bwd(s["u"], s["delta"], p["A"], s["B"], s["C"], s["dy"], self.ck, D=p.get("D"),
                       z=s["z"], delta_bias=p.get("delta_bias"), delta_softplus=True,
                       workspace=self.bws, out=s["g"])
            if self.allreduce is not None:
                self.allreduce(s["pgrad"])
            ev = torch.cuda.Event()
            ev.record(self.s_comp)
            self.comp_done[slot] = ev
        # ---- copy-out
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(self.comp_done[slot])
            host_out["y"].copy_(s["y"], non_blocking=True)
            for k in ("du", "ddelta", "dz", "dB", "dC", "dA", "dD", "ddelta_bias"):
                if s["g"][k] is not None and host_out.get(k) is not None:
                    host_out[k].copy_(s["g"][k], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(self.s_out)
            self.out_done[slot] = ev
        self.k += 1

    def first_copy_stream(self) -> torch.cuda.Stream:
        """The stream the first work of the next step is issued on (for timing events)."""
        return self.s_in

    def last_copy_stream(self) -> torch.cuda.Stream:
        """The stream the last work of a step is issued on (for timing events)."""
        return self.s_out

    def synchronize(self) -> None:
        for st in (self.s_in, self.s_comp, self.s_out):
            st.synchronize()

    @staticmethod
    def host_buffers(batch: int, dim: int, seqlen: int, dtype: torch.dtype,
                     dstate: int = ops.DSTATE, with_z: bool = True):
        """Pinned host tensors for one step's inputs and outputs (uninitialised)."""
        shp = (batch, dim, seqlen)
        hin = {k: torch.empty(shp, dtype=dtype, pin_memory=True) for k in ("u", "delta", "dy")}
        hin["z"] = torch.empty(shp, dtype=dtype, pin_memory=True) if with_z else None
        hin["B"] = torch.empty(batch, dstate, seqlen, dtype=dtype, pin_memory=True)
        hin["C"] = torch.empty(batch, dstate, seqlen, dtype=dtype, pin_memory=True)
        hout = {k: torch.empty(shp, dtype=dtype, pin_memory=True) for k in ("y", "du", "ddelta")}
        hout["dz"] = torch.empty(shp, dtype=dtype, pin_memory=True) if with_z else None
        hout["dB"] = torch.empty(batch, dstate, seqlen, dtype=torch.float32, pin_memory=True)
        hout["dC"] = torch.empty(batch, dstate, seqlen, dtype=torch.float32, pin_memory=True)
        hout["dA"] = torch.empty(dim, dstate, dtype=torch.float32, pin_memory=True)
        hout["dD"] = torch.empty(dim, dtype=torch.float32, pin_memory=True)
        hout["ddelta_bias"] = torch.empty(dim, dtype=torch.float32, pin_memory=True)
        return hin, hout
