"""Launch-failure injection (SS_FAIL_LAUNCH): every entry point that would
launch returns SS_ERR_CUDA with nothing enqueued, and the next call without the
variable works.  The failure is made on the host; no GPU fault is involved."""
import os

import pytest
import torch

from selective_state_space_11_b200 import inputs as gen
from selective_state_space_11_b200 import ops

pytestmark = pytest.mark.gpu


@pytest.fixture
def inject():
    os.environ["SS_FAIL_LAUNCH"] = "1"
    yield
    os.environ.pop("SS_FAIL_LAUNCH", None)


def _inputs():
    return {k: (None if v is None else v.cuda())
            for k, v in gen.make_inputs(2, 64, 16, 200, "f32", 901).items()}


def test_injected_launch_failure_is_reported_and_enqueues_nothing(inject):
    p = _inputs()
    y = torch.full_like(p["u"], float("nan"))
    with pytest.raises(ops.SSError) as ei:
        ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                   delta_bias=p["delta_bias"], out=(y, None, None), checkpoints=False)
    assert ei.value.status == 5 and "SS_FAIL_LAUNCH" in str(ei.value)   # SS_ERR_CUDA
    torch.cuda.synchronize()
    assert torch.isnan(y).all()                                      # nothing ran
    st = torch.zeros(2, 64, 16, device="cuda")
    with pytest.raises(ops.SSError):
        ops.ss_state_update(st, p["u"][..., 0].contiguous(), p["delta"][..., 0].contiguous(),
                            p["A"], p["B"][..., 0].contiguous(), p["C"][..., 0].contiguous())
    os.environ.pop("SS_FAIL_LAUNCH")
    y2, _, ck = ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                           delta_bias=p["delta_bias"])
    torch.cuda.synchronize()
    assert torch.isfinite(y2).all()
    os.environ["SS_FAIL_LAUNCH"] = "1"
    with pytest.raises(ops.SSError) as ei:
        ops.ss_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], p["dy"], ck, D=p["D"], z=p["z"],
                   delta_bias=p["delta_bias"])
    assert ei.value.status == 5


def test_zero_disables_injection():
    os.environ["SS_FAIL_LAUNCH"] = "0"
    try:
        p = _inputs()
        y, _, _ = ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"])
        torch.cuda.synchronize()
        assert torch.isfinite(y).all()
    finally:
        os.environ.pop("SS_FAIL_LAUNCH", None)
