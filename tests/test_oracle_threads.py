"""The oracle on all host cores (bench.py's CPU baseline): slices of the
(batch, channel) rows run by the unchanged sequential C code on separate
threads, with the sums across rows added in slice order, equal the sequential
oracle to fp64 rounding of those sums, for any thread count."""
import numpy as np
import pytest

import oracle
from selective_state_space_11_b200 import inputs as gen


@pytest.mark.parametrize("threads", [1, 3, 8])
def test_threads_equal_sequential(threads):
    p = gen.make_inputs(2, 64, 16, 200, "f32", 1000)
    q = {k: gen.as_f64(v) for k, v in p.items()}
    kw = dict(D=q["D"], z=q["z"], delta_bias=q["delta_bias"])
    y, fs, ck = oracle.ss_fwd(q["u"], q["delta"], q["A"], q["B"], q["C"], **kw)
    g = oracle.ss_bwd(q["u"], q["delta"], q["A"], q["B"], q["C"], q["dy"], **kw)
    y2, fs2, ck2, g2, used = oracle.ss_fwd_bwd_threads(q["u"], q["delta"], q["A"], q["B"], q["C"],
                                                       q["dy"], threads=threads, **kw)
    assert used == threads
    # rows are independent: per-row outputs are the same bits
    assert np.array_equal(y2, y) and np.array_equal(fs2, fs) and np.array_equal(ck2, ck)
    for k in ("du", "ddelta", "dz"):
        assert np.array_equal(g2[k], g[k]), k
    # sums across rows: same terms, another order of fp64 additions
    for k in ("dA", "dB", "dC", "dD", "dbias"):
        err = np.max(np.abs(g2[k] - g[k]) / (1 + np.abs(g[k])))
        assert err <= 1e-12, (k, err)


def test_host_cores_is_the_affinity_mask():
    import os
    assert oracle.host_cores() == len(os.sched_getaffinity(0))
