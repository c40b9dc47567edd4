"""Launch overlap (programmatic dependent launch) changes when kernels start, never what
they compute: with it on and off the outputs of every step are bitwise equal (on a B200)."""
import pytest
import torch

from patch_diffusion_unet_b200 import configs, inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg", [configs.get(1), configs.get(1, batch=2), configs.get(4)],
                         ids=["config1", "config1-b2", "config4"])
def test_overlap_on_off_bitwise_equal(cfg):
    from patch_diffusion_unet_b200 import dfp
    wl = inputs.SyntheticWorkload(cfg)
    weights = dict(wl.weights, context=wl.context) if wl.context is not None else wl.weights
    a, b = dfp.DisplacedPatchBlock(cfg), dfp.DisplacedPatchBlock(cfg)
    a.load_weights(weights)
    b.load_weights(weights)
    a.set_launch_overlap(True)
    b.set_launch_overlap(False)
    for t, s in wl.schedule()[:8]:
        x = inputs.to_torch(wl.x(t), "bf16").cuda()
        a.step(x, t, s)
        b.step(x, t, s)
        assert torch.equal(a.output(), b.output()), f"step {t}"
    a.check_device()
    b.check_device()
    a.close()
    b.close()
