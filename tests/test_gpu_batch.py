"""Parity of the guidance batch (B images per layer step) on a B200: the CUDA path
through the C ABI against the CPU oracle's batch, every image of every step.

The batch shares the weights and the step schedule only ("阅读论文1" paper-reading
blog, Implementation details: guidance scale 5; project README, Benchmarks:
--no_split_batch); each image keeps its own GroupNorm statistics, halo rows, K/V
context and, for the transformer stage, its own text context.  Same bars as the
single-image tests: rel-L2 <= 1e-5 (fp32) and <= 2e-2 (bf16) per step and stage.
"""
import numpy as np
import pytest
import torch

import oracle
from patch_diffusion_unet_b200 import configs, inputs
from tests.parity_util import TOL, host, rel_l2, run_parity

pytestmark = pytest.mark.gpu

STAGES = ("y", "y1", "h", "t", "q", "k", "v", "o")


def _assert(results, tol, stages=STAGES):
    for r in results:
        for s in stages:
            if s in r:
                assert r[s][0] <= tol, f"step {r['step']} stage {s}: rel-L2 {r[s][0]:.3e} > {tol} (max-abs {r[s][1]:.3e})"
        if "halo_ok" in r:
            assert r["halo_ok"], f"step {r['step']}: halo rows are not the expected copies"


@pytest.mark.parametrize("gn_mode,context", [(0, 0), (1, 0), (0, 1)], ids=["corrected", "stale_others", "naive"])
def test_config0_fp32_batch2(gn_mode, context):
    cfg = configs.get(0, batch=2)
    _assert(run_parity(cfg, cfg["steps"], gn_mode=gn_mode, context=context), TOL["f32"])


BATCHED = [
    # patch token counts not multiples of 128: image 1's K/V start mid-tile (row 960)
    dict(name="r40-b2", H=24, W=40, C=128, n_patches=3, gn_groups=8, gn_eps=1e-5, heads=2, head_dim=64,
         dtype="bf16", block="res_attn", steps=5, n_sync=2, batch=2),
    # three images, one row per patch
    dict(name="r1-b3", H=4, W=64, C=128, n_patches=4, gn_groups=8, gn_eps=1e-5, heads=2, head_dim=64,
         dtype="bf16", block="res_attn", steps=5, n_sync=2, batch=3),
    # N = 1: every patch is a whole image
    dict(name="n1-b2", H=16, W=32, C=192, n_patches=1, gn_groups=8, gn_eps=1e-5, heads=3, head_dim=64,
         dtype="bf16", block="res_attn", steps=4, n_sync=1, batch=2),
]


@pytest.mark.parametrize("cfg", BATCHED, ids=[c["name"] for c in BATCHED])
@pytest.mark.parametrize("family", [0, 1], ids=["tcgen05", "simt"])
def test_ragged_bf16_batch(cfg, family):
    _assert(run_parity(cfg, cfg["steps"], family=family, random_affine=True), TOL["bf16"])


def test_config1_batch2_first_steps_all_stages():
    cfg = configs.get(1, batch=2)
    _assert(run_parity(cfg, 7), TOL["bf16"])


def test_config1_batch2_whole_unit_rounds():
    """Two images with the attention's large-map split forced (K/V budget of one byte): the
    320 units (2 images x 4 patches x 10 heads x 4 pairs) make two whole rounds and a tail."""
    cfg = configs.get(1, batch=2)
    _assert(run_parity(cfg, 4, kv_budget=1), TOL["bf16"])


def test_batch_image0_matches_single_image_run():
    """Image 0 of a batch is the single-image workload: its output agrees with the
    single-image handle's at the bf16 bar (the launch shapes differ, so not bitwise)."""
    from patch_diffusion_unet_b200 import dfp
    cfg1, cfg2 = configs.get(1), configs.get(1, batch=2)
    wl1, wl2 = inputs.SyntheticWorkload(cfg1), inputs.SyntheticWorkload(cfg2)
    a, b = dfp.DisplacedPatchBlock(cfg1), dfp.DisplacedPatchBlock(cfg2)
    a.load_weights(wl1.weights)
    b.load_weights(wl2.weights)
    L = cfg1["H"] * cfg1["W"]
    for t, s in wl1.schedule()[:8]:
        a.step(inputs.to_torch(wl1.x(t), "bf16").cuda(), t, s)
        b.step(inputs.to_torch(wl2.x(t), "bf16").cuda(), t, s)
        ya, yb = host(a.output()), host(b.output())
        assert rel_l2(yb[:L], ya) <= 5e-3, f"step {t}"
    a.check_device()
    b.check_device()
    a.close()
    b.close()


STAGE = dict(name="stage-small-b2", H=16, W=32, C=128, n_patches=4, gn_groups=8, gn_eps=1e-5, heads=2,
             head_dim=64, dtype="bf16", block="sdxl_stage", steps=5, n_sync=2, n_xformer=2,
             ffn_inner=256, ctx_len=13, ctx_dim=96, batch=2)


def test_stage_batch2_own_contexts():
    """Two images with different text contexts through the transformer stage: every
    sub-layer stream of both images, and the cross-attention delta of each image (which
    only its own context can produce)."""
    from patch_diffusion_unet_b200 import dfp
    cfg = STAGE
    scale = {f"xf{b}.attn2.to_out.weight": 30.0 for b in range(2)}
    wl = inputs.SyntheticWorkload(cfg, weight_scale=scale, random_affine=True)
    assert wl.context.shape == (2, 13, 96)
    blk = dfp.DisplacedPatchBlock(cfg)
    blk.load_weights(dict(wl.weights, context=wl.context))
    orc = oracle.make_block(cfg, wl.weights, wl.context)
    B, H, W, C = 2, cfg["H"], cfg["W"], cfg["C"]
    names = ["resnet"] + [f"xf{b}.{n}" for b in range(2) for n in ("sa", "ca", "out")]
    for t, s in wl.schedule():
        x = wl.x(t)
        blk.step(inputs.to_torch(x, "bf16").cuda(), t, s)
        blk.check_device()
        ref = orc.step(x, t, s)
        g = {n: host(blk.buffer(n)).reshape(B, H, W, C) for n in names}
        for n in names:
            assert rel_l2(g[n], ref[n]) <= TOL["bf16"], f"step {t} {n}"
        for b in range(2):
            for xb in range(2):
                d_gpu = g[f"xf{xb}.ca"][b] - g[f"xf{xb}.sa"][b]
                d_ref = ref[f"xf{xb}.ca"][b] - ref[f"xf{xb}.sa"][b]
                assert rel_l2(d_gpu, d_ref) <= 3e-2, f"step {t} image {b} xf{xb} cross-attention delta"
    blk.close()


def test_pipelined_host_steps_batch2():
    from patch_diffusion_unet_b200 import dfp
    cfg = configs.get(1, batch=2)
    wl = inputs.SyntheticWorkload(cfg)
    a, b = dfp.DisplacedPatchBlock(cfg), dfp.DisplacedPatchBlock(cfg)
    a.load_weights(wl.weights)
    b.load_weights(wl.weights)
    sched = wl.schedule()[:7]
    xs = [inputs.to_torch(wl.x(t), "bf16").pin_memory() for t, _ in sched]
    ys = [torch.empty(2 * cfg["H"] * cfg["W"], cfg["C"], dtype=torch.bfloat16).pin_memory() for _ in sched]
    for i, (t, s) in enumerate(sched):
        b.step_host_async(xs[i], ys[i], t, s)
    b.synchronize()
    for i, (t, s) in enumerate(sched):
        a.step(xs[i].cuda(), t, s)
        assert torch.equal(a.output().cpu(), ys[i]), f"step {t}"
    a.close()
    b.close()
