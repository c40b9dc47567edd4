"""The allocation-free GroupNorm entry point (dfp_group_norm_noalloc), called
through the C ABI, against the same GroupNorm computed inside the regular layer
step (dfp_step, read back with dfp_copy_out).

It serves callers that cannot allocate device memory when they need the op, so
its scratch is a fixed array inside the library; two calls in a row check that
nothing left in that shared scratch by the first call leaks into the second.
This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from patch_diffusion_unet_b200 import configs, inputs

pytestmark = pytest.mark.gpu


def _rel(a, b):
    a = a.double().cpu()
    b = b.double().cpu()
    return float((a - b).norm() / b.norm())


def test_noalloc_group_norm_matches_layer_step_two_calls():
    from patch_diffusion_unet_b200 import dfp
    cfg = configs.get(1)
    H, W, C, N, G = cfg["H"], cfg["W"], cfg["C"], cfg["n_patches"], cfg["gn_groups"]
    R = H // N
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    blk = dfp.DisplacedPatchBlock(cfg)
    blk.load_weights(wl.weights)
    stream = torch.cuda.current_stream()
    gamma = torch.from_numpy(wl.weights["gn1.weight"]).float().cuda()
    beta = torch.from_numpy(wl.weights["gn1.bias"]).float().cuda()
    y = torch.empty(H * W, C, dtype=torch.bfloat16, device="cuda")
    fresh = [torch.empty(N * G * 2, device="cuda") for _ in range(2)]
    mr = torch.empty(N * G * 2, device="cuda")
    for t, is_sync in ((0, 1), (1, 0)):            # a sync call, then a displaced call
        x = inputs.to_torch(wl.x(t), "bf16").cuda()
        blk.step(x, t, is_sync)
        stale = None if is_sync else ctypes.c_void_p(fresh[0].data_ptr())
        st = dfp.LIB.dfp_group_norm_noalloc(
            ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()), dfp.BF16, H, W, C, N, G,
            cfg["gn_eps"], ctypes.c_void_p(gamma.data_ptr()), ctypes.c_void_p(beta.data_ptr()), stale,
            dfp.GN_CORRECTED, 1, ctypes.c_void_p(fresh[t].data_ptr()), ctypes.c_void_p(mr.data_ptr()),
            ctypes.c_void_p(stream.cuda_stream))
        assert st == dfp.OK, dfp.LIB.dfp_group_norm_noalloc_error().decode()
        torch.cuda.synchronize()
        ref_y = blk.buffer("slab").view(N, R + 2, W, C)[:, 1:R + 1].reshape(H * W, C)
        ref_mr = blk.buffer("gn1")
        assert _rel(y, ref_y) <= 2e-2
        assert _rel(mr, ref_mr) <= 2e-2
        blk.check_device()
    blk.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from patch_diffusion_unet_b200 import dfp
    null = ctypes.c_void_p(16)                      # never dereferenced: the size check fails first
    # one patch, 256 groups over a 64x64 map: 148 blocks x 256 groups x 2 partial sums > 64960
    st = dfp.LIB.dfp_group_norm_noalloc(null, null, dfp.BF16, 64, 64, 4096, 1, 256, 1e-5, null, null, None,
                                        dfp.GN_CORRECTED, 1, null, null, None)
    assert st == dfp.E_ARG
    assert "scratch" in dfp.LIB.dfp_group_norm_noalloc_error().decode()
