"""Failure detection on the GPU without a fault: a bounded wait that nothing satisfies
ends with an error code the host reads, and the context stays usable."""
import ctypes

import pytest

from patch_diffusion_unet_b200 import configs
from tests.parity_util import TOL, run_parity

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_with_a_code_and_the_context_survives():
    from patch_diffusion_unet_b200 import dfp
    code, cycles = ctypes.c_int(0), ctypes.c_longlong(0)
    assert dfp.LIB.dfp_selftest_wait_timeout(ctypes.byref(code), ctypes.byref(cycles)) == dfp.OK
    assert code.value == 1                        # "a TMA stage never filled"
    assert 1e9 < cycles.value < 1e10              # the ~4e9-clock limit, about 2 s
    # the same process and context still run layer steps correctly
    for r in run_parity(configs.get(0), 3):
        assert r["y"][0] <= TOL["f32"], f"step {r['step']}: rel-L2 {r['y'][0]:.3e}"


# ---------------------------------------------------------------- injected allocation failure
# DFP_FAULT_ALLOC_AFTER=k makes every library allocation after the first k fail as if the
# device were out of memory (a host-side fault: no GPU is driven into one).

def _with_fault(k):
    import os

    class _Env:
        def __enter__(self):
            os.environ["DFP_FAULT_ALLOC_AFTER"] = str(k)

        def __exit__(self, *exc):
            os.environ.pop("DFP_FAULT_ALLOC_AFTER", None)
    return _Env()


@pytest.mark.parametrize("k", [0, 3, 12])
@pytest.mark.parametrize("cid", [1, 4], ids=["layer", "stage"])
def test_create_reports_nomem_and_frees_everything(k, cid):
    import torch
    from patch_diffusion_unet_b200 import dfp
    cfg = configs.get(cid)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    with _with_fault(k):
        with pytest.raises(dfp.DfpError) as ei:
            dfp.DisplacedPatchBlock(cfg)
    assert ei.value.status == dfp.E_NOMEM
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0      # every allocation made before the failure was freed
    blk = dfp.DisplacedPatchBlock(cfg)                # and without the fault the same call succeeds
    blk.close()


def test_pipelined_host_step_set_up_fails_then_retries():
    """The pipelined host-buffer step allocates its staging buffers on first use: a failed
    set-up reports DFP_E_NOMEM and leaves nothing half-built, so the next call sets up and
    runs the step, with the same output as the device-buffer step."""
    import numpy as np
    import torch
    from patch_diffusion_unet_b200 import dfp, inputs
    cfg = configs.get(1)
    wl = inputs.SyntheticWorkload(cfg)
    a, b = dfp.DisplacedPatchBlock(cfg), dfp.DisplacedPatchBlock(cfg)
    a.load_weights(wl.weights)
    b.load_weights(wl.weights)
    x0 = inputs.to_torch(wl.x(0), "bf16")
    x1 = inputs.to_torch(wl.x(1), "bf16")
    y = torch.empty(cfg["H"] * cfg["W"], cfg["C"], dtype=torch.bfloat16).pin_memory()
    a.step(x0.cuda(), 0, 1)
    b.step(x0.cuda(), 0, 1)
    xp = x1.pin_memory()
    for k in (0, 1, 3):
        with _with_fault(k):
            with pytest.raises(dfp.DfpError) as ei:
                a.step_host_async(xp, y, 1, 0)
        assert ei.value.status == dfp.E_NOMEM
    a.step_host_async(xp, y, 1, 0)
    a.synchronize()
    b.step(x1.cuda(), 1, 0)
    assert np.array_equal(y.float().numpy(), b.output().float().cpu().numpy())
    a.check_device()
    a.close()
    b.close()
