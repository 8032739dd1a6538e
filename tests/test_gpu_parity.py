"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Small cases are compared in full; the named layer-shaped workloads are run at
full size in the same launch configuration the benchmark uses and checked on
sampled channels (plus the complete dB, dC of one batch row).
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_11_b200 import inputs as gen
from selective_state_space_11_b200 import ops
from tolerances import TOL, assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda"


def to_dev(p):
    return {k: (None if v is None else v.to(DEV)) for k, v in p.items()}


def f64(t):
    return gen.as_f64(t)


def gpu_fwd(p, sp=True):
    return ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                      delta_bias=p["delta_bias"], delta_softplus=sp)


def gpu_bwd(p, ck, sp=True):
    return ops.ss_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], p["dy"], ck, D=p["D"],
                      z=p["z"], delta_bias=p["delta_bias"], delta_softplus=sp)


def orc_fwd(p, sp=True):
    return oracle.ss_fwd(f64(p["u"]), f64(p["delta"]), f64(p["A"]), f64(p["B"]), f64(p["C"]),
                         D=f64(p["D"]), z=f64(p["z"]), delta_bias=f64(p["delta_bias"]),
                         delta_softplus=sp)


def orc_bwd(p, sp=True):
    return oracle.ss_bwd(f64(p["u"]), f64(p["delta"]), f64(p["A"]), f64(p["B"]), f64(p["C"]),
                         f64(p["dy"]), D=f64(p["D"]), z=f64(p["z"]),
                         delta_bias=f64(p["delta_bias"]), delta_softplus=sp)


def check_case(bsz, dim, L, dtype="f32", seed=0, sp=True, bwd=True, **flags):
    p = gen.make_inputs(bsz, dim, 16, L, dtype, seed, **flags)
    if not sp:  # keep Delta = delta + bias >= 0 without the softplus
        p["delta"] = p["delta"].abs() * 0.05
        if p["delta_bias"] is not None:
            p["delta_bias"] = p["delta_bias"].abs() * 0.01
    pd = to_dev(p)
    y, fs, ck = gpu_fwd(pd, sp)
    ry, rfs, rck = orc_fwd(p, sp)
    tf, tg = TOL[(dtype, "fwd")], TOL[(dtype, "grad")]
    n = assert_close(f64(y), ry, tf, "y")
    n += assert_close(f64(fs), rfs, tf, "final_state")
    n += assert_close(f64(ck), rck, tf, "checkpoints")
    if bwd:
        g = gpu_bwd(pd, ck, sp)
        r = orc_bwd(p, sp)
        for k_gpu, k_ref in [("du", "du"), ("ddelta", "ddelta"), ("dA", "dA"), ("dB", "dB"),
                             ("dC", "dC"), ("dD", "dD"), ("ddelta_bias", "dbias")]:
            n += assert_close(f64(g[k_gpu]), r[k_ref], tg, k_gpu)
        if p["z"] is not None:
            n += assert_close(f64(g["dz"]), r["dz"], tg, "dz")
    torch.cuda.synchronize()
    return n


# ------------------------------------------------------------- small cases --
@pytest.mark.parametrize("L", [200, 1, 64])
def test_tiny_workload(L):
    w = gen.WORKLOADS["tiny"]
    assert check_case(w.batch, w.dim, L, w.dtype, w.seed) > 0


@pytest.mark.parametrize("flags,sp", [
    (dict(), True), (dict(), False), (dict(with_z=False), True), (dict(with_D=False), True),
    (dict(with_bias=False), True), (dict(with_z=False, with_D=False, with_bias=False), False)])
def test_flag_grid(flags, sp):
    assert check_case(2, 8, 70, "f32", 5, sp=sp, **flags) > 0


@pytest.mark.parametrize("bsz,dim,L", [
    (1, 1, 1), (1, 1, 63), (2, 3, 64), (3, 3, 65), (1, 65, 200), (3, 64, 129), (2, 33, 7)])
def test_edge_shapes(bsz, dim, L):
    assert check_case(bsz, dim, L, "f32", 7 + L) > 0


def test_batch_rows_are_independent():
    """Batch-distinct data: each row's output depends only on its own B, C."""
    p = to_dev(gen.make_inputs(3, 5, 16, 90, "f32", 21))
    y, _, _ = gpu_fwd(p)
    for b in range(3):
        q = {k: v for k, v in p.items()}
        for k in ("u", "delta", "z", "B", "C", "dy"):
            q[k] = p[k][b:b + 1].contiguous()
        yb, _, _ = gpu_fwd(q)
        assert_close(f64(yb[0]), f64(y[b]), 1e-6, f"batch row {b} alone vs in batch")
    assert y.shape == (3, 5, 90)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_half_precision_small(dtype):
    assert check_case(2, 96, 300, dtype, 3) > 0


def test_per_channel_path():
    """Enough channels to fill the GPU: the per-channel path, fp32 and bf16."""
    path, nseg = ops.fwd_path(2, 2400, 130)
    assert (path, nseg) == (0, 1)
    assert check_case(2, 2400, 130, "f32", 11, bwd=False) > 0
    assert check_case(2, 2400, 96, "bf16", 12, bwd=True) > 0


# Enough channels (batch * d_inner >= 128 per SM) for the two-channel forward
# and backward kernels; ragged d_inner (not a multiple of 16) and ragged L.
PAIR_SHAPES = [(2, 9500, 70, "f32"), (2, 9496, 72, "bf16"), (1, 19000, 137, "bf16")]


@pytest.mark.parametrize("bsz,dim,L,dtype", PAIR_SHAPES)
def test_channel_pair_kernels(bsz, dim, L, dtype):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert bsz * dim >= 128 * sms, "shape must reach the channel-pair kernels"
    assert check_case(bsz, dim, L, dtype, 81 + L) > 0


def test_channel_pair_kernels_flags():
    assert check_case(2, 9500, 72, "bf16", 91, sp=False, with_z=False, with_D=False) > 0


def test_channel_pair_outputs_stay_inside_their_buffers():
    """Staged du / ddelta / dz rows of the pair walk land inside NaN-guarded buffers."""
    bsz, dim, L = 2, 9500, 72
    p = to_dev(gen.make_inputs(bsz, dim, 16, L, "bf16", 93))
    y, fs, ck = gpu_fwd(p)
    G = 64
    n = bsz * dim * L
    bufs = {k: torch.full((n + 2 * G,), float("nan"), device=DEV, dtype=torch.bfloat16)
            for k in ("du", "ddelta", "dz")}
    out = {k: b[G:G + n].view(bsz, dim, L) for k, b in bufs.items()}
    ops.ss_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], p["dy"], ck, D=p["D"], z=p["z"],
               delta_bias=p["delta_bias"], out=out)
    torch.cuda.synchronize()
    for k, b in bufs.items():
        assert torch.isnan(b[:G]).all() and torch.isnan(b[-G:]).all(), k
        assert torch.isfinite(out[k]).all(), k


def test_chunk_parallel_path_microbench():
    """The pages' microbenchmark shape (B=1, D=16, L=32768): chunk-parallel."""
    w = gen.WORKLOADS["microbench"]
    path, nseg = ops.fwd_path(w.batch, w.dim, w.seqlen)
    assert path == 1 and nseg > 1
    assert check_case(w.batch, w.dim, w.seqlen, w.dtype, w.seed, bwd=False) > 0


def test_chunk_parallel_ragged_segments():
    """Segments that do not divide L, ragged last chunk."""
    path, nseg = ops.fwd_path(1, 40, 64 * 37 + 5)
    assert path == 1 and nseg > 1
    assert check_case(1, 40, 64 * 37 + 5, "f32", 13) > 0


@pytest.mark.parametrize("dim,L,cache", [
    (200, 64 * 20 + 9, 1), (16, 64 * 300 + 1, 4), (12, 64 * 600 + 3, 16), (8, 64 * 2300 + 5, 32),
    (4, 64 * 4500 + 7, 0)])
def test_chunk_parallel_carry_scan_slabs(dim, L, cache):
    """Segment counts that take each register-cache size of the carry scan:
    up to 32 warps of 4 slabs each split the segments into contiguous slabs,
    and a slab of more than 32 segments re-reads its maps from global memory
    (cache 0).
    Ragged rows and an initial state (composed in at the first slab); the
    forward is checked in full against the oracle."""
    path, nseg = ops.fwd_path(1, dim, L)
    assert path == 1 and nseg > 1
    slabs = 4 * min(32, -(-nseg // 4))
    per = -(-nseg // slabs)  # segments per slab
    taken = next((c for c in (1, 4, 16, 32) if per <= c), 0)
    if taken != cache:
        pytest.skip(f"this device splits L into {nseg} segments ({per} per slab), not the case meant")
    p = gen.make_inputs(1, dim, 16, L, "f32", 17 + dim)
    h0 = gen.make_state(1, dim, 16, 17 + dim)
    pd = to_dev(p)
    y, fs, ck = ops.ss_fwd(pd["u"], pd["delta"], pd["A"], pd["B"], pd["C"], D=pd["D"], z=pd["z"],
                           delta_bias=pd["delta_bias"], h0=h0.to(DEV))
    ry, rfs, rck = oracle.ss_fwd(f64(p["u"]), f64(p["delta"]), f64(p["A"]), f64(p["B"]), f64(p["C"]),
                                 D=f64(p["D"]), z=f64(p["z"]), delta_bias=f64(p["delta_bias"]),
                                 h0=f64(h0))
    tf = TOL[("f32", "fwd")]
    assert_close(f64(y), ry, tf, "y")
    assert_close(f64(fs), rfs, tf, "final_state")
    assert_close(f64(ck), rck, tf, "checkpoints")


def test_chunk_parallel_in_cuda_graph():
    """The chunk-parallel chain (local pass, carry scan, full pass; the last two
    launched with programmatic dependent launch) captured in a CUDA graph and
    replayed gives bitwise the eager results, call after call on reused
    buffers."""
    bsz, dim, L = 1, 16, 64 * 200 + 11
    path, nseg = ops.fwd_path(bsz, dim, L)
    assert path == 1 and nseg > 1
    p = to_dev(gen.make_inputs(bsz, dim, 16, L, "f32", 61))
    h0 = gen.make_state(bsz, dim, 16, 61).to(DEV)
    ry, rfs, rck = ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                              delta_bias=p["delta_bias"], h0=h0)
    ws = torch.empty(max(16, ops.lib().ss_fwd_workspace_size(bsz, dim, 16, L)), device=DEV,
                     dtype=torch.uint8)
    y, fs, ck = torch.empty_like(ry), torch.empty_like(rfs), torch.empty_like(rck)

    def call():
        ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                   delta_bias=p["delta_bias"], h0=h0, out=(y, fs, ck), workspace=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(3):
            call()
    for _ in range(2):
        for t in (y, fs, ck):
            t.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, ry) and torch.equal(fs, rfs) and torch.equal(ck, rck)
    del graph


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_state_update(dtype):
    bsz, dim = 3, 70
    p = gen.make_inputs(bsz, dim, 16, 1, dtype, 31)
    tok = {k: p[k][..., 0].contiguous() for k in ("u", "delta", "z", "B", "C")}
    st0 = torch.randn(bsz, dim, 16, generator=torch.Generator().manual_seed(4))
    rst, ry = oracle.ss_state_update(st0.double().numpy(), f64(tok["u"]), f64(tok["delta"]),
                                     f64(p["A"]), f64(tok["B"]), f64(tok["C"]), D=f64(p["D"]),
                                     z=f64(tok["z"]), delta_bias=f64(p["delta_bias"]))
    st = st0.to(DEV)
    y = ops.ss_state_update(st, *(tok[k].to(DEV) for k in ("u", "delta")), p["A"].to(DEV),
                            tok["B"].to(DEV), tok["C"].to(DEV), D=p["D"].to(DEV),
                            z=tok["z"].to(DEV), delta_bias=p["delta_bias"].to(DEV))
    assert_close(f64(y), ry, TOL[(dtype, "fwd")], "decode y")
    assert_close(f64(st), rst, TOL[(dtype, "fwd")], "decode state")


def test_prefill_then_decode_equals_full_forward():
    bsz, dim, L1, k = 2, 48, 1000, 24
    p = gen.make_inputs(bsz, dim, 16, L1 + k, "f32", 41)
    pd = to_dev(p)
    y_full, fs_full, _ = gpu_fwd(pd)
    pre = dict(pd)
    for key in ("u", "delta", "z", "B", "C", "dy"):
        pre[key] = pd[key][..., :L1].contiguous()
    _, st, _ = gpu_fwd(pre)
    ys = []
    for t in range(L1, L1 + k):
        ys.append(ops.ss_state_update(st, pd["u"][..., t].contiguous(),
                                      pd["delta"][..., t].contiguous(), pd["A"],
                                      pd["B"][..., t].contiguous(), pd["C"][..., t].contiguous(),
                                      D=pd["D"], z=pd["z"][..., t].contiguous(),
                                      delta_bias=pd["delta_bias"]))
    y_dec = torch.stack(ys, dim=-1)
    ry, rfs, _ = orc_fwd(p)
    assert_close(f64(y_dec), ry[..., L1:], TOL[("f32", "fwd")], "decode vs oracle")
    assert_close(f64(st), rfs, TOL[("f32", "fwd")], "decode state vs oracle")
    assert_close(f64(y_dec), f64(y_full[..., L1:]), TOL[("f32", "fwd")], "decode vs gpu fwd")


@pytest.mark.parametrize("bsz,dim,L", [(2, 300, 333), (2, 9500, 200)])
def test_bitwise_deterministic(bsz, dim, L):
    p = to_dev(gen.make_inputs(bsz, dim, 16, L, "bf16", 51))
    y1, f1, c1 = gpu_fwd(p)
    g1 = gpu_bwd(p, c1)
    y2, f2, c2 = gpu_fwd(p)
    g2 = gpu_bwd(p, c2)
    assert torch.equal(y1, y2) and torch.equal(f1, f2) and torch.equal(c1, c2)
    for k in g1:
        if g1[k] is not None:
            assert torch.equal(g1[k], g2[k]), k


def test_outputs_stay_inside_their_buffers():
    """Outputs written into NaN-filled guard bands: the guards stay untouched."""
    bsz, dim, L = 2, 37, 150
    p = to_dev(gen.make_inputs(bsz, dim, 16, L, "f32", 61))
    G = 64
    ybuf = torch.full((bsz * dim * L + 2 * G,), float("nan"), device=DEV)
    fbuf = torch.full((bsz * dim * 16 + 2 * G,), float("nan"), device=DEV)
    nck = (L + 63) // 64
    cbuf = torch.full((bsz * dim * nck * 16 + 2 * G,), float("nan"), device=DEV)
    y = ybuf[G:G + bsz * dim * L].view(bsz, dim, L)
    fs = fbuf[G:G + bsz * dim * 16].view(bsz, dim, 16)
    ck = cbuf[G:G + bsz * dim * nck * 16].view(bsz, dim, nck, 16)
    ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
               delta_bias=p["delta_bias"], out=(y, fs, ck))
    for buf, inner in ((ybuf, y), (fbuf, fs), (cbuf, ck)):
        assert torch.isnan(buf[:G]).all() and torch.isnan(buf[-G:]).all()
        assert torch.isfinite(inner).all()


def test_workspace_too_small_is_an_error():
    p = to_dev(gen.make_inputs(1, 16, 16, 4096, "f32", 71))
    need = ops.lib().ss_fwd_workspace_size(1, 16, 16, 4096)
    assert need > 0
    ws = torch.empty(need - 16, device=DEV, dtype=torch.uint8)
    with pytest.raises(ops.SSError, match="SS_ERR_WORKSPACE"):
        import ctypes
        P = ctypes.c_void_p
        y = torch.empty_like(p["u"])
        ops._check(ops.lib().ss_fwd(1, 16, 16, 4096, 0, P(p["u"].data_ptr()),
                                    P(p["delta"].data_ptr()), None, P(p["A"].data_ptr()),
                                    P(p["B"].data_ptr()), P(p["C"].data_ptr()), None, None, 1,
                                    P(y.data_ptr()), None, None, P(ws.data_ptr()), need - 16,
                                    None))


def test_autograd_function_matches_bwd():
    p = to_dev(gen.make_inputs(2, 24, 16, 100, "f32", 81))
    leaves = {k: p[k].clone().requires_grad_(True) for k in ("u", "delta", "A", "B", "C", "D",
                                                             "z", "delta_bias")}
    y = ops.selective_scan_fn(leaves["u"], leaves["delta"], leaves["A"], leaves["B"],
                              leaves["C"], D=leaves["D"], z=leaves["z"],
                              delta_bias=leaves["delta_bias"], delta_softplus=True)
    (y * p["dy"]).sum().backward()
    r = orc_bwd({k: (v.cpu() if v is not None else None) for k, v in p.items()})
    for k, rk in [("u", "du"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"), ("C", "dC"),
                  ("D", "dD"), ("z", "dz"), ("delta_bias", "dbias")]:
        assert_close(f64(leaves[k].grad), r[rk], TOL[("f32", "grad")], "autograd " + k)


# ------------------------------------------- full-size layer workloads -----
def _sample_channels(bsz, dim, k, seed):
    rng = np.random.default_rng(seed)
    pts = {(0, 0), (bsz - 1, dim - 1), (0, dim - 1)}
    while len(pts) < k:
        pts.add((int(rng.integers(bsz)), int(rng.integers(dim))))
    return sorted(pts)


def _rows(p, b, d):
    q = {}
    for k in ("u", "delta", "z", "dy"):
        q[k] = None if p[k] is None else p[k][b:b + 1, d:d + 1]
    for k in ("B", "C"):
        q[k] = p[k][b:b + 1]
    q["A"] = p["A"][d:d + 1]
    q["D"] = None if p["D"] is None else p["D"][d:d + 1]
    q["delta_bias"] = None if p["delta_bias"] is None else p["delta_bias"][d:d + 1]
    return {k: (None if v is None else v.cpu()) for k, v in q.items()}


def _full_size(name, nsample, full_batch_row=True):
    w = gen.WORKLOADS[name]
    pd = gen.workload_inputs(name, device=DEV)
    y, fs, ck = gpu_fwd(pd)
    g = gpu_bwd(pd, ck)
    torch.cuda.synchronize()
    tf, tg = TOL[(w.dtype, "fwd")], TOL[(w.dtype, "grad")]
    n = 0
    for (b, d) in _sample_channels(w.batch, w.dim, nsample, w.seed):
        q = _rows(pd, b, d)
        ry, rfs, rck = orc_fwd(q)
        n += assert_close(f64(y[b, d]), ry[0, 0], tf, f"y[{b},{d}]")
        n += assert_close(f64(fs[b, d]), rfs[0, 0], tf, f"final[{b},{d}]")
        n += assert_close(f64(ck[b, d]), rck[0, 0], tf, f"ckpt[{b},{d}]")
        r = orc_bwd(q)
        for kg, kr in (("du", "du"), ("ddelta", "ddelta"), ("dz", "dz")):
            n += assert_close(f64(g[kg][b, d]), r[kr][0, 0], tg, f"{kg}[{b},{d}]")
    # parameter gradients of a sampled channel need every batch row
    for d in sorted({d for _, d in _sample_channels(w.batch, w.dim, 3, w.seed + 1)}):
        q = {k: None if pd[k] is None else pd[k].cpu() for k in pd}
        for k in ("u", "delta", "z", "dy"):
            q[k] = q[k][:, d:d + 1]
        for k in ("D", "delta_bias"):
            q[k] = q[k][d:d + 1]
        q["A"] = q["A"][d:d + 1]
        r = orc_bwd(q)
        n += assert_close(f64(g["dA"][d]), r["dA"][0], tg, f"dA[{d}]")
        n += assert_close(f64(g["dD"][d]), r["dD"][0], tg, f"dD[{d}]")
        n += assert_close(f64(g["ddelta_bias"][d]), r["dbias"][0], tg, f"dbias[{d}]")
    if full_batch_row:
        # channel sums: dB, dC of batch row 0 need every channel of that row
        q = {k: None if pd[k] is None else pd[k].cpu() for k in pd}
        for k in ("u", "delta", "z", "dy", "B", "C"):
            q[k] = q[k][0:1]
        r = orc_bwd(q)
        n += assert_close(f64(g["dB"][0]), r["dB"][0], tg, "dB[0]")
        n += assert_close(f64(g["dC"][0]), r["dC"][0], tg, "dC[0]")
    return n


def test_mamba130m_layer_full_size():
    assert _full_size("mamba130m_layer", 8) > 0


def test_mamba2p8b_layer_full_size():
    assert _full_size("mamba2.8b_layer", 6) > 0


def test_long_prefill_then_decode_full_size():
    w = gen.WORKLOADS["long_prefill_decode"]
    L, k = w.seqlen, w.decode_steps
    pd = gen.make_inputs(w.batch, w.dim, 16, L + k, w.dtype, w.seed, device=DEV, with_dy=False)
    pre = dict(pd)
    for key in ("u", "delta", "z", "B", "C"):
        pre[key] = pd[key][..., :L].contiguous()
    assert ops.fwd_path(w.batch, w.dim, L)[0] == 1
    _, st, _ = ops.ss_fwd(pre["u"], pre["delta"], pre["A"], pre["B"], pre["C"], D=pre["D"],
                          z=pre["z"], delta_bias=pre["delta_bias"], checkpoints=False)
    ys = []
    for t in range(L, L + k):
        ys.append(ops.ss_state_update(st, pd["u"][..., t].contiguous(),
                                      pd["delta"][..., t].contiguous(), pd["A"],
                                      pd["B"][..., t].contiguous(), pd["C"][..., t].contiguous(),
                                      D=pd["D"], z=pd["z"][..., t].contiguous(),
                                      delta_bias=pd["delta_bias"]))
    y_dec = torch.stack(ys, dim=-1)
    y_full, fs_full, _ = ops.ss_fwd(pd["u"], pd["delta"], pd["A"], pd["B"], pd["C"], D=pd["D"],
                                    z=pd["z"], delta_bias=pd["delta_bias"], checkpoints=False)
    tol = TOL[(w.dtype, "fwd")]
    assert_close(f64(y_dec), f64(y_full[..., L:]), tol, "decode vs one full forward")
    assert_close(f64(st), f64(fs_full), tol, "decode state vs full forward state")
    for (b, d) in _sample_channels(w.batch, w.dim, 4, w.seed):
        q = _rows(dict(pd, dy=None), b, d)
        ry, rfs, _ = orc_fwd(q)
        assert_close(f64(y_full[b, d]), ry[0, 0], tol, f"long y[{b},{d}]")
        assert_close(f64(y_dec[b, d]), ry[0, 0, L:], tol, f"decode y[{b},{d}]")
        assert_close(f64(st[b, d]), rfs[0, 0], tol, f"decode state[{b},{d}]")
