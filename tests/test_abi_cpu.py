"""The C-ABI library loads and exports every declared symbol; host-side argument
checks reject bad configurations before any CUDA call (CPU only, no GPU needed)."""
import ctypes
import os
import re

import pytest

from patch_diffusion_unet_b200 import configs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^DFP_API\s+[\w\s\*]+?\b(dfp_\w+)\s*\(", text, re.M))
    return names


def test_library_exports_every_declared_symbol():
    from patch_diffusion_unet_b200 import dfp
    declared = _declared()
    assert declared, "no declarations found"
    missing = [n for n in declared if not hasattr(dfp.LIB, n)]
    assert not missing, missing
    assert set(dfp.EXPORTED) <= declared


def _create(**over):
    from patch_diffusion_unet_b200 import dfp
    cfg = configs.get(1, **over)
    c = dfp.make_config(cfg)
    h = ctypes.c_void_p()
    st = dfp.LIB.dfp_create(ctypes.byref(c), None, ctypes.byref(h))
    return st, dfp.LIB.dfp_last_error(None).decode(), h


@pytest.mark.parametrize("over,frag", [
    (dict(n_patches=3), "multiple of n_patches"),
    (dict(gn_groups=33), "multiple of gn_groups"),
    (dict(head_dim=32), "head_dim"),
    (dict(heads=9), "heads * head_dim"),
    (dict(H=0), "positive"),
    (dict(gn_eps=-1.0), "gn_eps"),
    (dict(n_patches=16, gn_groups=32), "<= 256"),
])
def test_create_rejects_bad_config(over, frag):
    from patch_diffusion_unet_b200 import dfp
    st, msg, h = _create(**over)
    assert st == dfp.E_ARG
    assert frag in msg
    assert not h.value


def test_create_rejects_fp32_stage_and_bad_stage_sizes():
    from patch_diffusion_unet_b200 import dfp
    h = ctypes.c_void_p()
    c = dfp.make_config(configs.get(4, dtype="f32"))
    assert dfp.LIB.dfp_create(ctypes.byref(c), None, ctypes.byref(h)) == dfp.E_UNSUPPORTED
    c = dfp.make_config(configs.get(4, ffn_inner=100))
    assert dfp.LIB.dfp_create(ctypes.byref(c), None, ctypes.byref(h)) == dfp.E_ARG
    c = dfp.make_config(configs.get(4, n_xformer=3))
    assert dfp.LIB.dfp_create(ctypes.byref(c), None, ctypes.byref(h)) == dfp.E_ARG


def test_null_arguments():
    from patch_diffusion_unet_b200 import dfp
    L = dfp.LIB
    assert L.dfp_create(None, None, None) == dfp.E_ARG
    assert L.dfp_destroy(None) == dfp.OK
    assert L.dfp_step(None, None, 0, 1) == dfp.E_ARG
    assert L.dfp_check_device(None) == dfp.E_ARG
    assert L.dfp_launches_per_step(None) == -1
    assert L.dfp_set_launch_overlap(None, 1) == dfp.E_ARG
    assert L.dfp_set_kernel_family(None, 0) == dfp.E_ARG
    assert L.dfp_synchronize(None) == dfp.E_ARG
    assert L.dfp_step_host_async(None, None, None, 0, 1) == dfp.E_ARG
    assert isinstance(L.dfp_last_error(None), bytes)


def _noalloc(x, y, stale, fresh, mr, H=64, W=64, C=640, N=4, G=32):
    from patch_diffusion_unet_b200 import dfp
    p = ctypes.c_void_p
    return dfp.LIB.dfp_group_norm_noalloc(p(x), p(y), dfp.BF16, H, W, C, N, G, 1e-5, p(1 << 20), p(2 << 20),
                                          None if stale is None else p(stale), dfp.GN_CORRECTED, 1, p(fresh),
                                          None if mr is None else p(mr), None)


@pytest.mark.parametrize("case,frag", [
    # the displaced call reads stale_moments after writing fresh_moments: one buffer for
    # both would silently turn every displaced call into the synchronous statistics
    ("stale_is_fresh", "stale_moments and fresh_moments overlap"),
    ("stale_overlaps_fresh", "stale_moments and fresh_moments overlap"),
    ("y_is_x", "x and y overlap"),
    ("y_overlaps_x", "x and y overlap"),
    ("mean_rstd_is_fresh", "mean_rstd and fresh_moments overlap"),
    ("mean_rstd_is_stale", "mean_rstd and stale_moments overlap"),
])
def test_noalloc_rejects_overlapping_buffers(case, frag):
    """Host checks of dfp_group_norm_noalloc, before anything touches a GPU (the
    addresses are never dereferenced)."""
    from patch_diffusion_unet_b200 import dfp
    x, y = 1 << 30, 2 << 30                       # 64x64x640 bf16 maps: 5.2 MB each
    stale, fresh, mr = 3 << 30, 4 << 30, 5 << 30  # [4, 32, 2] fp32: 1 KiB each
    if case == "stale_is_fresh":
        stale = fresh
    elif case == "stale_overlaps_fresh":
        stale = fresh + 512
    elif case == "y_is_x":
        y = x
    elif case == "y_overlaps_x":
        y = x + 64 * 64 * 640 * 2 - 16
    elif case == "mean_rstd_is_fresh":
        mr = fresh
    elif case == "mean_rstd_is_stale":
        mr = stale
    assert _noalloc(x, y, stale, fresh, mr) == dfp.E_ARG
    assert frag in dfp.LIB.dfp_group_norm_noalloc_error().decode()


def test_noalloc_adjacent_buffers_pass_the_overlap_checks():
    """Buffers that only touch (one ends where the next starts) do not overlap: the call
    gets past every overlap check and stops at the scratch-size check that follows them
    (one patch of 64x64x4096 in 256 groups needs more partial sums than the fixed
    scratch holds), still before any CUDA call."""
    from patch_diffusion_unet_b200 import dfp
    H, W, C, N, G = 64, 64, 4096, 1, 256
    mb, nb = H * W * C * 2, N * G * 2 * 4
    x, fresh = 1 << 30, 4 << 30
    st = _noalloc(x, x + mb, fresh - nb, fresh, fresh + nb, H=H, W=W, C=C, N=N, G=G)
    assert st == dfp.E_ARG
    assert "scratch" in dfp.LIB.dfp_group_norm_noalloc_error().decode()
