"""Sequence sharding on CPU ranks (gloo, world size 2 and 3).

Each rank takes one contiguous segment of L for every batch row and channel
and runs dist.seq_sharded_forward / seq_sharded_backward, the same
orchestration the GPU path uses, with the fp64 oracle standing in for the
library's segment kernels: the forward and backward of a segment, its state
transition P (from its definition: the end state of the segment run with
u = 0 from h0 = 1) and the chain of segment states.  The exchange goes over
gloo collectives.  Stitched together, the segments must reproduce the oracle
run over the whole sequence: y, the final state, every gradient and dh0.
"""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest
import torch

from selective_state_space_11_b200 import dist as ssdist
from selective_state_space_11_b200 import inputs as gen

BSZ, DIM, N, L, SEED = 2, 6, 16, 90, 91


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleKernels:
    """The segment steps of sequence sharding, computed by the fp64 oracle."""

    def __init__(self, oracle):
        self.o = oracle

    @staticmethod
    def _np(t):
        return None if t is None else t.numpy()

    def fwd(self, seg, h0):
        y, fs, ck = self.o.ss_fwd(seg["u"], seg["delta"], seg["A"], seg["B"], seg["C"], D=seg["D"], z=seg["z"],
                                  delta_bias=seg["delta_bias"], delta_softplus=seg["delta_softplus"],
                                  h0=self._np(h0))
        return torch.from_numpy(y), torch.from_numpy(fs), torch.from_numpy(ck)

    def bwd(self, seg, dy, checkpoints, h0, dfinal):
        g = self.o.ss_bwd(seg["u"], seg["delta"], seg["A"], seg["B"], seg["C"], dy, D=seg["D"], z=seg["z"],
                          delta_bias=seg["delta_bias"], delta_softplus=seg["delta_softplus"], h0=self._np(h0),
                          dfinal=self._np(dfinal))
        out = {k: (None if v is None else torch.from_numpy(np.ascontiguousarray(v))) for k, v in g.items()}
        out["ddelta_bias"] = out.pop("dbias")
        return out

    def decay(self, seg):
        u0 = np.zeros_like(seg["u"])
        ones = np.ones((seg["u"].shape[0], seg["u"].shape[1], seg["A"].shape[1]))
        _, fs, _ = self.o.ss_fwd(u0, seg["delta"], seg["A"], seg["B"], seg["C"], delta_bias=seg["delta_bias"],
                                 delta_softplus=seg["delta_softplus"], h0=ones)
        return torch.from_numpy(fs)

    def chain(self, P, E, reverse):
        out = torch.empty_like(P)
        S = P.shape[0]
        h = torch.zeros_like(P[0])
        order = range(S - 1, -1, -1) if reverse else range(S)
        prev = None
        for s in order:
            if prev is not None:
                h = P[prev] * h + E[prev]
            out[s] = h
            prev = s
        return out


def _inputs():
    p = gen.make_inputs(BSZ, DIM, N, L, "f32", SEED)
    f = gen.as_f64
    q = {k: (None if p[k] is None else f(p[k])) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias", "dy")}
    rng = np.random.default_rng(SEED)
    q["h0"] = rng.standard_normal((BSZ, DIM, N))
    q["dfinal"] = rng.standard_normal((BSZ, DIM, N))
    return q


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q = _inputs()
        lo, hi = ssdist.shard_seq(L, rank, world)
        seg = {k: q[k][..., lo:hi].copy() for k in ("u", "delta", "B", "C", "z")}
        seg.update(A=q["A"], D=q["D"], delta_bias=q["delta_bias"], delta_softplus=True)
        dy = q["dy"][..., lo:hi].copy()
        kern = OracleKernels(oracle)
        gather = lambda t: ssdist.all_gather_stacked(t)
        allreduce = lambda t: dist.all_reduce(t)
        y, end, ck, h_in, P = ssdist.seq_sharded_forward(seg, torch.from_numpy(q["h0"]), rank, world, gather, kern)
        g = ssdist.seq_sharded_backward(seg, dy, ck, h_in, P, torch.from_numpy(q["dfinal"]), rank, world,
                                        gather, allreduce, kern)
        out.put((rank, lo, hi, y.numpy(), end.numpy(),
                 {k: (None if v is None else v.numpy()) for k, v in g.items()}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_sharding_matches_the_whole_sequence(world):
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = sorted([q.get(timeout=180) for _ in range(world)], key=lambda r: r[0])
    for pr in procs:
        pr.join(60)
        assert pr.exitcode == 0

    x = _inputs()
    y, fs, _ = oracle.ss_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                             delta_bias=x["delta_bias"], h0=x["h0"])
    full = oracle.ss_bwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dy"], D=x["D"], z=x["z"],
                         delta_bias=x["delta_bias"], h0=x["h0"], dfinal=x["dfinal"])
    close = lambda a, b: np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-9)
    covered = []
    for rank, lo, hi, ys, end, g in res:
        covered.extend(range(lo, hi))
        close(ys, y[..., lo:hi])
        for k in ("du", "ddelta", "dz", "dB", "dC"):
            close(g[k], full[k][..., lo:hi])
        close(g["dA"], full["dA"])
        close(g["dD"], full["dD"])
        close(g["ddelta_bias"], full["dbias"])
        if rank == world - 1:
            close(end, fs)
        if rank == 0:
            close(g["dh0"], full["dh0"])
    assert covered == list(range(L))


def test_shard_seq_partition():
    for length in (1, 7, 64, 90):
        for world in range(1, 5):
            spans = [ssdist.shard_seq(length, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == length
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c and b >= a
