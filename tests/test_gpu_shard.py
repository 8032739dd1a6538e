"""Sequence sharding on the GPU: the segment transition and chain kernels
against their definitions, and the sharded forward and backward, with ranks
emulated by host threads on one GPU, against the fp64 oracle run over the
whole sequence.  The threads meet only on the host (a barrier around each
exchange); no kernel waits on another."""
import threading

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_11_b200 import dist as ssdist
from selective_state_space_11_b200 import inputs as gen
from selective_state_space_11_b200 import ops
from tolerances import TOL, assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
f64 = gen.as_f64


@pytest.mark.parametrize("dtype,softplus", [("f32", True), ("bf16", True), ("f32", False)])
def test_segment_decay_is_the_segment_state_transition(dtype, softplus):
    """P equals the end state of the segment run with u = 0 from h0 = 1."""
    p = gen.make_inputs(3, 40, 16, 333, dtype, 501)
    if not softplus:  # Delta = delta + bias must stay positive without softplus
        p["delta"] = p["delta"].abs()
        p["delta_bias"] = p["delta_bias"].abs()
    P = ops.segment_decay(p["delta"].to(DEV), p["A"].to(DEV), p["delta_bias"].to(DEV), softplus)
    u0 = np.zeros(p["u"].shape)
    _, ref, _ = oracle.ss_fwd(u0, f64(p["delta"]), f64(p["A"]), f64(p["B"]), f64(p["C"]),
                              delta_bias=f64(p["delta_bias"]), delta_softplus=softplus,
                              h0=np.ones((3, 40, 16)))
    assert_close(f64(P), ref, TOL[("f32", "fwd")], "P")


@pytest.mark.parametrize("reverse", [False, True])
def test_state_chain_matches_its_recurrence(reverse):
    g = torch.Generator().manual_seed(7)
    S, shape = 5, (2, 33, 16)
    P = torch.rand((S,) + shape, generator=g)
    E = torch.randn((S,) + shape, generator=g)
    out = ops.state_chain(P.to(DEV), E.to(DEV), None, reverse=reverse).cpu().double()
    ref = torch.empty((S,) + shape, dtype=torch.float64)
    h = torch.zeros(shape, dtype=torch.float64)
    order = list(range(S - 1, -1, -1)) if reverse else list(range(S))
    for i, s in enumerate(order):
        if i:
            prev = order[i - 1]
            h = P[prev].double() * h + E[prev].double()
        ref[s] = h
    assert_close(out.numpy(), ref.numpy(), 1e-5, "chain")


class _Threads:
    """Collectives for ranks emulated by host threads on one GPU."""

    def __init__(self, world):
        self.slots = [None] * world
        self.bar = threading.Barrier(world)

    def gather(self, rank, t):
        self.slots[rank] = t
        self.bar.wait()
        out = torch.stack(self.slots)
        self.bar.wait()
        return out

    def allreduce(self, rank, t):
        t.copy_(self.gather(rank, t.clone()).sum(0))


@pytest.mark.parametrize("world,dtype", [(3, "f32"), (4, "bf16")])
def test_sequence_sharded_forward_backward(world, dtype):
    bsz, dim, N, L = 2, 64, 16, 600
    p = gen.make_inputs(bsz, dim, N, L, dtype, 611)
    rng = np.random.default_rng(611)
    h0 = torch.from_numpy(rng.standard_normal((bsz, dim, N))).float()
    dfinal = torch.from_numpy(rng.standard_normal((bsz, dim, N))).float()
    ops.lib()  # load the library before the threads start
    group = _Threads(world)
    res, errs = [None] * world, []

    def run(rank):
        try:
            lo, hi = ssdist.shard_seq(L, rank, world)
            cut = lambda t: t[..., lo:hi].contiguous().to(DEV)
            seg = {k: cut(p[k]) for k in ("u", "delta", "B", "C", "z")}
            seg.update(A=p["A"].to(DEV), D=p["D"].to(DEV), delta_bias=p["delta_bias"].to(DEV),
                       delta_softplus=True)
            y, end, ck, h_in, P = ssdist.seq_sharded_forward(seg, h0.to(DEV), rank, world,
                                                             lambda t: group.gather(rank, t))
            g = ssdist.seq_sharded_backward(seg, cut(p["dy"]), ck, h_in, P, dfinal.to(DEV), rank, world,
                                            lambda t: group.gather(rank, t),
                                            lambda t: group.allreduce(rank, t))
            torch.cuda.synchronize()
            res[rank] = (lo, hi, y, end, g)
        except Exception as e:  # surfaced below
            errs.append(e)
            group.bar.abort()

    threads = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(300)
    assert not errs, errs
    x = {k: (None if p[k] is None else f64(p[k])) for k in p}
    y, fs, _ = oracle.ss_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                             delta_bias=x["delta_bias"], h0=f64(h0))
    full = oracle.ss_bwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dy"], D=x["D"], z=x["z"],
                         delta_bias=x["delta_bias"], h0=f64(h0), dfinal=f64(dfinal))
    tf, tg = TOL[(dtype, "fwd")], TOL[(dtype, "grad")]
    for rank, (lo, hi, ys, end, g) in enumerate(res):
        assert_close(f64(ys), y[..., lo:hi], tf, f"y rank {rank}")
        for k in ("du", "ddelta", "dz", "dB", "dC"):
            assert_close(f64(g[k]), full[k][..., lo:hi], tg, f"{k} rank {rank}")
        assert_close(f64(g["dA"]), full["dA"], tg, f"dA rank {rank}")
        assert_close(f64(g["dD"]), full["dD"], tg, f"dD rank {rank}")
        assert_close(f64(g["ddelta_bias"]), full["dbias"], tg, f"dbias rank {rank}")
    assert_close(f64(res[-1][3]), fs, tf, "final state")
    assert_close(f64(res[0][4]["dh0"]), full["dh0"], tg, "dh0")
