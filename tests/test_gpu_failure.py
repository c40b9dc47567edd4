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
