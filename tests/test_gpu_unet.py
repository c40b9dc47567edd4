"""The multi-level UNet (DFP_BLOCK_UNET) on a B200 against the CPU oracle's displaced UNet
(oracle/unet_oracle.py): the predicted noise of single UNet steps, synchronous and
displaced, and whole DDIM runs, at the bf16 bar (2e-2 relative L2)."""
import numpy as np
import pytest
import torch

from oracle import unet_oracle as uo
from patch_diffusion_unet_b200 import configs, inputs
from tests.parity_util import TOL, host, rel_l2

pytestmark = pytest.mark.gpu

SMALL = dict(name="unet-32x32-n2", H=32, W=32, C=64, n_patches=2, gn_groups=8, gn_eps=1e-5, heads=1, head_dim=64,
             dtype="bf16", block="unet", steps=6, n_sync=2, widths=(64, 128, 256), latent_c=4, ctx_len=5, ctx_dim=16,
             ddim_train_steps=1000, beta_start=0.00085, beta_end=0.012)


def _pair(cfg, gn_mode=0):
    from patch_diffusion_unet_b200 import dfp
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    blk = dfp.DisplacedPatchBlock(cfg, gn_mode=gn_mode)
    blk.load_weights(dict(wl.weights, context=wl.context))
    orc = uo.DisplacedUNet(cfg, wl.weights, wl.context, gn_mode=["corrected", "stale_others", "sync", "separate"][gn_mode])
    return wl, blk, orc


def _latents(cfg, n, seed=3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((cfg["H"], cfg["W"], cfg["latent_c"]))
    out = []
    for _ in range(n):
        out.append(inputs.round_to(x, "bf16"))
        x = 0.95 * x + 0.05 * rng.standard_normal(x.shape)
    return out


@pytest.mark.parametrize("gn_mode", [0, 1], ids=["corrected", "stale_others"])
def test_small_unet_steps(gn_mode):
    cfg = SMALL
    wl, blk, orc = _pair(cfg, gn_mode)
    taus = uo.ddim_timesteps(cfg["steps"], 1000)
    for t, (x, tau) in enumerate(zip(_latents(cfg, cfg["steps"]), taus)):
        is_sync = int(t < cfg["n_sync"])
        blk.set_timestep(float(tau))
        blk.step(inputs.to_torch(x, "bf16").cuda(), t, is_sync)
        blk.check_device()
        want = orc.step(x, t, is_sync, tau)
        got = host(blk.output()).reshape(cfg["H"], cfg["W"], 4)
        err = rel_l2(got, want["eps"])
        assert err <= TOL["bf16"], f"step {t}: eps rel-L2 {err:.3e}"
        for name, ref in (("s0", want["s0"]), ("s1", want["s1"]), ("mid", want["mid"]), ("up0", want["up0"])):
            g = host(blk.buffer(name)).reshape(ref.shape)
            assert rel_l2(g, ref) <= TOL["bf16"], f"step {t}: {name} rel-L2 {rel_l2(g, ref):.3e}"
    blk.close()


def test_small_unet_ddim_run():
    cfg = SMALL
    wl, blk, orc = _pair(cfg)
    xT = wl.latent()
    n, n_sync = 6, 2
    out = blk.ddim_sample(torch.from_numpy(np.ascontiguousarray(xT, np.float32)).cuda(), n, n_sync)
    torch.cuda.synchronize()
    blk.check_device()
    want = uo.ddim_sample(orc, xT, n, n_sync)[-1]
    assert rel_l2(host(out), want) <= TOL["bf16"]
    blk.close()


def test_full_size_unet_displaced_step():
    """The 1024 px UNet (latent 128x128, 8 patches per level): GPU steps 0-5, the first five
    synchronous; the oracle joins at step 4 (synchronous) and checks steps 4 and 5."""
    cfg = configs.get(5)
    wl, blk, _ = _pair(cfg)
    orc = uo.DisplacedUNet(cfg, wl.weights, wl.context)
    taus = uo.ddim_timesteps(50, 1000)
    for t, x in enumerate(_latents(cfg, 6)):
        is_sync = int(t < cfg["n_sync"])
        blk.set_timestep(float(taus[t]))
        blk.step(inputs.to_torch(x, "bf16").cuda(), t, is_sync)
        blk.check_device()
        if t < 4:
            continue
        want = orc.step(x, t - 4, is_sync, taus[t])["eps"]
        err = rel_l2(host(blk.output()).reshape(want.shape), want)
        assert err <= TOL["bf16"], f"step {t}: eps rel-L2 {err:.3e}"
    blk.close()
