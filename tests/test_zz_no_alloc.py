"""The allocation-free GroupNorm entry point (dfp_group_norm_noalloc), called
through the C ABI.

It serves callers that cannot allocate device memory when they need the op (a
fixed memory pool that bans the CUDA allocator, a pre-planned region, a host
path that must not take allocator locks), so its scratch is a fixed array
inside the library.  Each case runs two calls in a row -- a synchronous call,
then a displaced one fed the first call's moments -- so that anything the first
call leaves in the shared scratch would show in the second.  The output is
compared with the CPU oracle's displaced GroupNorm (fp32 storage at 1e-5, bf16
at 2e-2 relative L2) and, for the layer step's own GroupNorm configuration,
with the GroupNorm inside dfp_step.  This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from patch_diffusion_unet_b200 import configs, inputs
from tests.parity_util import TOL, rel_l2

pytestmark = pytest.mark.gpu

MODES = {0: oracle.GN_CORRECTED, 1: oracle.GN_STALE_OTHERS, 2: oracle.GN_SYNC, 3: oracle.GN_SEPARATE}


def _call(dfp, x, y, dtype, cfg, gamma, beta, stale, mode, silu, fresh, mr):
    H, W, C, N, G = cfg["H"], cfg["W"], cfg["C"], cfg["n_patches"], cfg["gn_groups"]
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = dfp.LIB.dfp_group_norm_noalloc(
        ptr(x), ptr(y), dtype, H, W, C, N, G, cfg["gn_eps"], ptr(gamma), ptr(beta), ptr(stale), mode,
        int(silu), ptr(fresh), ptr(mr), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == dfp.OK, dfp.LIB.dfp_group_norm_noalloc_error().decode()


@pytest.mark.parametrize("cid", [0, 1], ids=["fp32-16x16x64", "bf16-64x64x640"])
@pytest.mark.parametrize("mode", [0, 1, 2, 3], ids=["corrected", "stale_others", "gn_sync", "gn_separate"])
@pytest.mark.parametrize("silu,keep_mr", [(True, True), (False, False)], ids=["silu", "no-silu-no-mean_rstd"])
def test_noalloc_matches_oracle_two_calls(cid, mode, silu, keep_mr):
    from patch_diffusion_unet_b200 import dfp
    cfg = configs.get(cid)
    H, W, C, N, G = cfg["H"], cfg["W"], cfg["C"], cfg["n_patches"], cfg["gn_groups"]
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    g_np, b_np = wl.weights["gn1.weight"], wl.weights["gn1.bias"]
    ref = oracle.DisplacedGroupNorm(N, G, cfg["gn_eps"], g_np, b_np, MODES[mode], silu=silu)
    gamma = torch.from_numpy(g_np).float().cuda()
    beta = torch.from_numpy(b_np).float().cuda()
    tdt = torch.bfloat16 if cfg["dtype"] == "bf16" else torch.float32
    code = dfp.BF16 if cfg["dtype"] == "bf16" else dfp.F32
    y = torch.empty(H * W, C, dtype=tdt, device="cuda")
    fresh = [torch.empty(N * G * 2, device="cuda") for _ in range(2)]   # alternate two buffers
    mr = torch.empty(N * G * 2, device="cuda") if keep_mr else None
    for t, is_sync in ((0, 1), (1, 0)):
        x_np = wl.x(t)
        x = inputs.to_torch(x_np, cfg["dtype"]).cuda()
        y.fill_(float("nan"))
        _call(dfp, x, y, code, cfg, gamma, beta, None if is_sync else fresh[0], mode, silu, fresh[t], mr)
        torch.cuda.synchronize()
        want = ref(x_np, is_sync)
        got = y.double().cpu().numpy().reshape(H, W, C)
        err = rel_l2(got, want)
        assert err <= TOL[cfg["dtype"]], f"step {t}: rel-L2 {err:.3e}"
        # this call's moments: (mean, variance) per (patch, group), what the next call reads
        raw = np.stack([oracle.group_moments(x_np[r0:r1], G) for r0, r1 in oracle.patch_bounds(H, N)])
        want_m = np.stack([raw[..., 0], raw[..., 1] - raw[..., 0] ** 2], axis=-1)
        assert rel_l2(fresh[t].double().cpu().numpy().reshape(N, G, 2), want_m) <= 1e-5
        if keep_mr:
            mu, var = ref.last
            want_mr = np.stack([mu, 1.0 / np.sqrt(var + cfg["gn_eps"])], axis=-1)
            assert rel_l2(mr.double().cpu().numpy().reshape(N, G, 2), want_mr) <= 1e-5


def test_noalloc_matches_layer_step_two_calls():
    """Same inputs as the layer step's first GroupNorm (GN1 + SiLU of dfp_step)."""
    from patch_diffusion_unet_b200 import dfp
    cfg = configs.get(1)
    H, W, C, N, G = cfg["H"], cfg["W"], cfg["C"], cfg["n_patches"], cfg["gn_groups"]
    R = H // N
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    blk = dfp.DisplacedPatchBlock(cfg)
    blk.load_weights(wl.weights)
    gamma = torch.from_numpy(wl.weights["gn1.weight"]).float().cuda()
    beta = torch.from_numpy(wl.weights["gn1.bias"]).float().cuda()
    y = torch.empty(H * W, C, dtype=torch.bfloat16, device="cuda")
    fresh = [torch.empty(N * G * 2, device="cuda") for _ in range(2)]
    mr = torch.empty(N * G * 2, device="cuda")
    for t, is_sync in ((0, 1), (1, 0)):
        x = inputs.to_torch(wl.x(t), "bf16").cuda()
        blk.step(x, t, is_sync)
        _call(dfp, x, y, dfp.BF16, cfg, gamma, beta, None if is_sync else fresh[0], dfp.GN_CORRECTED, True,
              fresh[t], mr)
        torch.cuda.synchronize()
        ref_y = blk.buffer("slab").view(N, R + 2, W, C)[:, 1:R + 1].reshape(H * W, C)
        assert rel_l2(y.double().cpu().numpy(), ref_y.double().cpu().numpy()) <= TOL["bf16"]
        assert rel_l2(mr.double().cpu().numpy(), blk.buffer("gn1").double().cpu().numpy()) <= 1e-5
        blk.check_device()
    blk.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from patch_diffusion_unet_b200 import dfp
    null = ctypes.c_void_p(16)                      # never dereferenced: the size check fails first
    # one patch, 256 groups over a 64x64 map: 148 blocks x 256 groups x 2 partial sums > 64960
    st = dfp.LIB.dfp_group_norm_noalloc(null, ctypes.c_void_p(1 << 30), dfp.BF16, 64, 64, 4096, 1, 256, 1e-5, null,
                                        null, None, dfp.GN_CORRECTED, 1, ctypes.c_void_p(2 << 30), None, None)
    assert st == dfp.E_ARG
    assert "scratch" in dfp.LIB.dfp_group_norm_noalloc_error().decode()
