"""The attention softmax's polynomial exponential, run on the B200 through the
test-only entry point dfp_selftest_exp2_poly (the same device code the softmax
inlines), against exp2 in fp64: relative error within the fit's bound of 7.5e-5
(plus fp32 evaluation rounding) over the softmax's input range [-125, 0], and
the bf16 value the softmax stores equal to the fp32 result truncated."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _run(x_np):
    from patch_diffusion_unet_b200 import dfp
    x = torch.from_numpy(x_np.astype(np.float32)).cuda()
    n = x.numel()
    y = torch.empty(n, dtype=torch.float32, device="cuda")
    yb = torch.empty(n + 1, dtype=torch.bfloat16, device="cuda")
    st = dfp.LIB.dfp_selftest_exp2_poly(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()),
                                        ctypes.c_void_p(yb.data_ptr()), n,
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == dfp.OK
    torch.cuda.synchronize()
    return y.cpu().numpy(), yb[:n].cpu().view(torch.int16).numpy().astype(np.uint16)


@pytest.mark.parametrize("n", [1_000_001, 1_000_000])   # odd and even: the last pair may be half
def test_exp2_poly_error_bound(n):
    x = np.linspace(-125.0, 0.0, n)
    x = np.concatenate([x, -np.arange(0, 125) - 0.5, [0.0, -0.5, -1e-7]]).astype(np.float32)
    y, yb = _run(x)
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 7.5e-5 + 4 * 2.0 ** -24, f"max relative error {rel.max():.3e} at x = {x[rel.argmax()]}"
    assert np.array_equal(yb, (y.view(np.uint32) >> 16).astype(np.uint16))


def test_exp2_poly_below_clamp_and_empty():
    from patch_diffusion_unet_b200 import dfp
    y, _ = _run(np.array([-126.0, -300.0, -1e30, -np.inf], np.float32))
    assert np.all(np.abs(y.astype(np.float64) / 2.0 ** -125 - 1.0) <= 7.5e-5)
    assert dfp.LIB.dfp_selftest_exp2_poly(None, None, None, 0, None) == dfp.OK
    assert dfp.LIB.dfp_selftest_exp2_poly(None, None, None, 4, None) == dfp.E_ARG
