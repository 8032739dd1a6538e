"""Host-resident steps with overlapped copies (streaming.HostStepPipeline):
every step's results, copied back to host memory, equal bit for bit those of
ss_fwd + ss_bwd called directly on device copies of the same inputs, also
when consecutive steps' copies and kernels overlap."""
import pytest
import torch

from selective_state_space_11_b200 import inputs as gen
from selective_state_space_11_b200 import ops
from selective_state_space_11_b200.streaming import HostStepPipeline

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("bsz,dim,L,dtype", [(2, 64, 200, "f32"), (2, 1016, 640, "bf16")])
def test_pipeline_matches_direct_calls(bsz, dim, L, dtype):
    steps = [gen.make_inputs(bsz, dim, 16, L, dtype, 900 + i) for i in range(4)]
    params = {k: steps[0][k].to(DEV) for k in ("A", "D", "delta_bias")}
    tdt = steps[0]["u"].dtype
    pipe = HostStepPipeline(bsz, dim, L, tdt, params, DEV)
    bufs = []
    for st in steps:
        hin, hout = HostStepPipeline.host_buffers(bsz, dim, L, tdt)
        for k in hin:
            hin[k].copy_(st[k])
        bufs.append((hin, hout))
        pipe.step(hin, hout)
    pipe.synchronize()
    for st, (hin, hout) in zip(steps, bufs):
        d = {k: (None if v is None else v.to(DEV)) for k, v in st.items()}
        y, _, ck = ops.ss_fwd(d["u"], d["delta"], params["A"], d["B"], d["C"], D=params["D"],
                              z=d["z"], delta_bias=params["delta_bias"])
        g = ops.ss_bwd(d["u"], d["delta"], params["A"], d["B"], d["C"], d["dy"], ck,
                       D=params["D"], z=d["z"], delta_bias=params["delta_bias"])
        torch.cuda.synchronize()
        assert torch.equal(hout["y"], y.cpu())
        for k in ("du", "ddelta", "dz", "dB", "dC", "dA", "dD", "ddelta_bias"):
            assert torch.equal(hout[k], g[k].cpu()), k
