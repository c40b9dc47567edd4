"""The guidance batch (B images, one layer step each) on the CPU: pins of the oracle's
batch against PyTorch's batched library routines, the input recipe, and the
host-side checks of the C ABI (no GPU needed).

A batch of images shares the weights and the step schedule and nothing else: the
classifier-free-guidance pair (conditional, unconditional; guidance scale 5,
"阅读论文1" paper-reading blog, Implementation details) that the project README's
benchmarks split across GPU groups unless --no_split_batch is given (README,
Benchmarks).  PyTorch's group_norm keeps statistics per sample and
scaled_dot_product_attention attends within each batch element, so a batched
full-map layer written with them is an independent statement of "no mixing".
"""
import ctypes

import numpy as np
import pytest

import oracle
from patch_diffusion_unet_b200 import configs, inputs
from tests import torch_ref

SMALL = dict(name="small", H=8, W=6, C=32, n_patches=4, gn_groups=4, gn_eps=1e-5, heads=4,
             head_dim=8, dtype="f32", block="res_attn", steps=4, n_sync=1, batch=2)
STAGE = dict(name="stage-small", H=8, W=4, C=32, n_patches=2, gn_groups=4, gn_eps=1e-5, heads=2,
             head_dim=16, dtype="f32", block="sdxl_stage", steps=3, n_sync=1, n_xformer=2,
             ffn_inner=48, ctx_len=5, ctx_dim=12, batch=2)


def _close(a, b, tol=1e-10):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape, (a.shape, b.shape)
    err = np.abs(a - b).max()
    scale = max(np.abs(b).max(), 1e-30)
    assert err <= tol * scale, f"max-abs {err} vs scale {scale}"


def _full(cfg, xs, wl):
    xs = np.asarray(xs, np.float64)
    if cfg["block"] == "res_attn":
        return torch_ref.res_attn_full_batched(xs, wl.weights, cfg)
    return torch_ref.sdxl_stage_full_batched(xs, wl.weights, np.asarray(wl.context, np.float64), cfg)


def test_batch_inputs_recipe():
    """Image 0 of a batch is the single-image workload; the other images are new draws."""
    wl1 = inputs.SyntheticWorkload(configs.get(STAGE, batch=1))
    wl3 = inputs.SyntheticWorkload(configs.get(STAGE, batch=3))
    for k in wl1.weights:
        assert np.array_equal(wl1.weights[k], wl3.weights[k])
    assert wl3.context.shape == (3, 5, 12) and np.array_equal(wl3.context[0], wl1.context)
    assert not np.array_equal(wl3.context[1], wl3.context[2])
    for t in range(3):
        x1, x3 = wl1.x(t), wl3.x(t)
        assert x3.shape == (3, 8, 4, 32)
        assert np.array_equal(x3[0], x1)
        assert not np.array_equal(x3[1], x3[0])


@pytest.mark.parametrize("cfg", [SMALL, configs.get(SMALL, batch=3, n_patches=2), STAGE],
                         ids=["res2", "res3-n2", "stage2"])
def test_batch_sync_step_equals_batched_full_layer(cfg):
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    blk = oracle.make_block(cfg, wl.weights, wl.context)
    x = wl.x(0)
    out = blk.step(x, 0, 1)
    ref = _full(cfg, x, wl)
    _close(out["y"], ref["y"])
    if cfg["block"] == "res_attn":
        for k in ("y1", "h", "t", "o"):
            _close(out[k], ref[k])


@pytest.mark.parametrize("mode", ["corrected", "stale_others"])
@pytest.mark.parametrize("cfg", [SMALL, STAGE], ids=["res", "stage"])
def test_batch_stale_equal_to_fresh_gives_batched_full_layer(cfg, mode):
    """A displaced step whose cache holds this very map is each image's full layer: the
    stale statistics and K/V of one image never stand in for another's."""
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    blk = oracle.make_block(cfg, wl.weights, wl.context, gn_mode=mode)
    x = wl.x(0)
    blk.step(x, 0, 1)
    out = blk.step(x, 1, 0)
    _close(out["y"], _full(cfg, x, wl)["y"])


def test_batch_images_do_not_interact():
    """Changing image 1's inputs leaves image 0's outputs unchanged at every step,
    displaced steps included."""
    cfg = SMALL
    wl_a = inputs.SyntheticWorkload(cfg)
    wl_b = inputs.SyntheticWorkload(cfg)
    blk_a = oracle.make_block(cfg, wl_a.weights)
    blk_b = oracle.make_block(cfg, wl_b.weights)
    for t, s in wl_a.schedule():
        xa = wl_a.x(t)
        xb = wl_b.x(t).copy()
        xb[1] = -2.0 * xb[1] + 0.5
        ya, yb = blk_a.step(xa, t, s)["y"], blk_b.step(xb, t, s)["y"]
        assert np.array_equal(ya[0], yb[0])
        assert np.abs(ya[1] - yb[1]).max() > 1e-3


def test_batch_of_one_image_each_matches_single_blocks():
    """Each image of the batch runs exactly the single-image step on its own input."""
    cfg = SMALL
    wl = inputs.SyntheticWorkload(cfg)
    blk = oracle.make_block(cfg, wl.weights)
    singles = [oracle.make_block(configs.get(cfg, batch=1), wl.weights) for _ in range(2)]
    for t, s in wl.schedule():
        x = wl.x(t)
        y = blk.step(x, t, s)["y"]
        for b in range(2):
            assert np.array_equal(y[b], singles[b].step(x[b], t, s)["y"])


# --------------------------------------------------------------------------- C ABI (host side)

def _create(cfg):
    from patch_diffusion_unet_b200 import dfp
    c = dfp.make_config(cfg)
    h = ctypes.c_void_p()
    st = dfp.LIB.dfp_create(ctypes.byref(c), None, ctypes.byref(h))
    return st, dfp.LIB.dfp_last_error(None).decode(), h


@pytest.mark.parametrize("over,frag", [
    (dict(batch=9), "batch must be"),
    (dict(batch=-1), "batch must be"),
    (dict(batch=8, H=4096, W=4096), "too large"),
])
def test_create_rejects_bad_batch(over, frag):
    from patch_diffusion_unet_b200 import dfp
    st, msg, h = _create(configs.get(1, **over))
    assert st == dfp.E_ARG and frag in msg and not h.value


def test_create_rejects_fp32_batch_past_the_simt_limit():
    from patch_diffusion_unet_b200 import dfp
    st, msg, h = _create(configs.get(0, batch=5, n_patches=16, gn_groups=8, H=16))
    assert st == dfp.E_ARG and "512" in msg and not h.value
