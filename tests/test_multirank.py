"""Multi-rank data parallelism on CPU (gloo, world size 2).

Each rank takes its batch rows, runs the fp64 oracle's backward on them, and
all-reduces the packed parameter gradients with the same helper the benchmark
uses over NCCL.  The result must equal the full-batch gradients, and the
per-row gradients must be unaffected by the sharding.
"""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest
import torch

from selective_state_space_11_b200 import dist as ssdist
from selective_state_space_11_b200 import inputs as gen


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, batch, q):
    import torch.distributed as dist

    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p = gen.make_inputs(batch, 12, 16, 70, "f32", 77)
        lo, hi = ssdist.shard_rows(batch, rank, world)
        f = lambda t: None if t is None else gen.as_f64(t)
        g = oracle.ss_bwd(f(p["u"][lo:hi]), f(p["delta"][lo:hi]), f(p["A"]), f(p["B"][lo:hi]),
                          f(p["C"][lo:hi]), f(p["dy"][lo:hi]), D=f(p["D"]), z=f(p["z"][lo:hi]),
                          delta_bias=f(p["delta_bias"]))
        buf, views = ssdist.param_grad_buffer(12, 16, "cpu")
        views["dA"].copy_(torch.from_numpy(g["dA"]))
        views["dD"].copy_(torch.from_numpy(g["dD"]))
        views["ddelta_bias"].copy_(torch.from_numpy(g["dbias"]))
        ssdist.allreduce_param_grads(buf)
        q.put((rank, lo, hi, buf.numpy().copy(), g["du"], g["dB"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("batch", [4, 3])
def test_batch_sharding_and_param_grad_allreduce(batch):
    import oracle
    oracle.build()
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, batch, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for pr in procs:
        pr.join(60)
        assert pr.exitcode == 0
    res.sort(key=lambda r: r[0])

    p = gen.make_inputs(batch, 12, 16, 70, "f32", 77)
    f = gen.as_f64
    full = oracle.ss_bwd(f(p["u"]), f(p["delta"]), f(p["A"]), f(p["B"]), f(p["C"]), f(p["dy"]),
                         D=f(p["D"]), z=f(p["z"]), delta_bias=f(p["delta_bias"]))
    expect = np.concatenate([full["dA"].ravel(), full["dD"], full["dbias"]])
    covered = []
    for rank, lo, hi, buf, du, dB in res:
        # every rank ends with the same, full-batch parameter gradients
        np.testing.assert_allclose(buf, expect, rtol=1e-6, atol=1e-6)
        # its own rows' gradients match the full-batch computation exactly
        np.testing.assert_allclose(du, full["du"][lo:hi], rtol=0, atol=0)
        np.testing.assert_allclose(dB, full["dB"][lo:hi], rtol=0, atol=0)
        covered.extend(range(lo, hi))
    assert covered == list(range(batch))


def test_shard_rows_partition():
    for batch in range(1, 9):
        for world in range(1, 5):
            spans = [ssdist.shard_rows(batch, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == batch
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c and b >= a
    with pytest.raises(ValueError):
        ssdist.shard_rows(4, 2, 2)
