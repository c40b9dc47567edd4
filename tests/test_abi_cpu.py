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
