"""Pins of the UNet oracle (oracle/unet_oracle.py) on the CPU, against what the pages and
the mathematics fix: a synchronous step, an N = 1 step and a step whose stale context
equals the fresh one are the whole network written with PyTorch's library routines
(strided conv2d, nearest interpolate, cat, group_norm, SDPA, layer_norm, GELU); the
stride-2 conv's halo is local; the DDIM update, its timesteps and schedule and the
timestep embedding meet closed forms."""
import numpy as np
import pytest

from oracle import unet_oracle as uo
from patch_diffusion_unet_b200 import configs, inputs
from tests import torch_ref

TINY = dict(name="unet-tiny", H=16, W=16, C=64, n_patches=2, gn_groups=8, gn_eps=1e-5, heads=1, head_dim=64,
            dtype="f32", block="unet", steps=6, n_sync=2, widths=(64, 128, 128), latent_c=4, ctx_len=5, ctx_dim=12,
            ddim_train_steps=1000, beta_start=0.00085, beta_end=0.012)
KEYS = ("eps", "mid", "s0", "s1", "up0")


def _close(a, b, tol=1e-10):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape, (a.shape, b.shape)
    err = np.abs(a - b).max()
    assert err <= tol * max(np.abs(b).max(), 1e-30), err


def _net(cfg, **kw):
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    return wl, uo.DisplacedUNet(cfg, wl.weights, wl.context, **kw)


def test_sync_step_equals_the_library_network():
    wl, net = _net(TINY)
    x = wl.latent().astype(np.float64)
    out = net.step(x, 0, 1, 981)
    ref = torch_ref.unet_full(x, wl.weights, wl.context, TINY, 981)
    for k in KEYS:
        _close(out[k], ref[k])


def test_n1_displaced_steps_equal_the_library_network():
    cfg = dict(TINY, n_patches=1)
    wl, net = _net(cfg)
    rng = np.random.default_rng(4)
    for t, tau in enumerate((981, 961, 941)):
        x = rng.standard_normal((16, 16, 4))
        _close(net.step(x, t, int(t == 0), tau)["eps"], torch_ref.unet_full(x, wl.weights, wl.context, cfg, tau)["eps"])


@pytest.mark.parametrize("N", [2, 4])
def test_stale_equal_to_fresh_gives_the_library_network(N):
    cfg = dict(TINY, n_patches=N, H=32, W=16)
    wl, net = _net(cfg)
    x = np.random.default_rng(5).standard_normal((32, 16, 4))
    net.step(x, 0, 1, 501)
    out = net.step(x, 1, 0, 501)            # displaced, with this very map in every cache
    ref = torch_ref.unet_full(x, wl.weights, wl.context, cfg, 501)
    for k in KEYS:
        _close(out[k], ref[k])


def test_displaced_step_differs_from_sync():
    wl, net = _net(TINY)
    rng = np.random.default_rng(6)
    net.step(rng.standard_normal((16, 16, 4)), 0, 1, 981)
    x = rng.standard_normal((16, 16, 4))
    y = net.step(x, 1, 0, 961)["eps"]
    assert np.abs(y - torch_ref.unet_full(x, wl.weights, wl.context, TINY, 961)["eps"]).max() > 1e-6


def test_downsample_halo_is_the_row_above_the_patch():
    rng = np.random.default_rng(7)
    N, H, W, C = 4, 16, 6, 3
    R = H // N
    wgt, b = rng.standard_normal((5, C, 3, 3)), rng.standard_normal(5)
    prev, y = rng.standard_normal((H, W, C)), rng.standard_normal((H, W, C))
    base = uo.DisplacedDownsample(N, wgt, b)
    base(prev, True)
    ref = base(y, False)
    # full-map strided conv of the assembled per-patch inputs (row above from the stale map)
    import torch
    import torch.nn.functional as F
    for p in range(N):
        band = np.concatenate([prev[p * R - 1:p * R] if p else np.zeros((1, W, C)), y[p * R:(p + 1) * R]])
        out = F.conv2d(torch.from_numpy(np.pad(band, ((0, 0), (0, 0), (0, 0)))).permute(2, 0, 1)[None],
                       torch.from_numpy(wgt), torch.from_numpy(b), stride=2, padding=(0, 1))[0].permute(1, 2, 0).numpy()
        _close(ref[p * R // 2:(p + 1) * R // 2], out)
    # only the row above a patch is read from the stale map
    for row in range(H):
        p2 = prev.copy()
        p2[row] += 1.0
        d = uo.DisplacedDownsample(N, wgt, b)
        d(p2, True)
        changed = np.abs(d(y, False) - ref).max(axis=(1, 2)) > 0
        feeds = row % R == R - 1 and row < H - 1            # the last row of a patch feeds the next
        assert changed.any() == feeds, row
        if feeds:
            assert np.flatnonzero(changed).tolist() == [(row + 1) // 2]


def test_ddim_step_recovers_the_noised_sample():
    """With the true noise as the prediction, one DDIM step moves x_t = sqrt(ab) x0 +
    sqrt(1 - ab) e exactly to sqrt(ab_prev) x0 + sqrt(1 - ab_prev) e."""
    rng = np.random.default_rng(8)
    x0, e = rng.standard_normal(50), rng.standard_normal(50)
    for ab, ab_prev in ((0.3, 0.5), (0.0047, 0.0052), (0.99, 1.0)):
        xt = np.sqrt(ab) * x0 + np.sqrt(1 - ab) * e
        _close(uo.ddim_step(xt, e, ab, ab_prev), np.sqrt(ab_prev) * x0 + np.sqrt(1 - ab_prev) * e)


def test_schedule_timesteps_and_embedding_closed_forms():
    taus = uo.ddim_timesteps(50, 1000)
    assert taus.tolist() == list(range(981, 0, -20))
    ab = uo.alphas_cumprod(1000, 0.00085, 0.012)
    assert ab[0] == pytest.approx(1 - 0.00085, rel=1e-15)
    assert ab[1] == pytest.approx((1 - 0.00085) * (1 - (np.sqrt(0.00085) + (np.sqrt(0.012) - np.sqrt(0.00085)) / 999) ** 2))
    assert np.all(np.diff(ab) < 0) and ab[-1] == pytest.approx(ab[-2] * (1 - 0.012))
    e0 = uo.timestep_embedding(0.0, 8)
    assert e0.tolist() == [1.0] * 4 + [0.0] * 4
    e1 = uo.timestep_embedding(1.0, 8)
    assert e1[0] == pytest.approx(np.cos(1.0)) and e1[4] == pytest.approx(np.sin(1.0))
    assert e1[1] == pytest.approx(np.cos(10000 ** -0.25))


def test_ddim_loop_runs_and_stays_finite():
    cfg = TINY
    wl, net = _net(cfg)
    xs = uo.ddim_sample(net, wl.latent(), 6, 2)
    assert len(xs) == 6 and all(np.isfinite(x).all() for x in xs)


def test_full_size_workload_shapes():
    cfg = configs.get(5)
    specs = dict(inputs.weight_specs(cfg))
    assert specs["up1.resnet.conv1.weight"] == (640, 1920, 3, 3)
    assert specs["up0.resnet.conv_shortcut.weight"] == (320, 960)
    assert specs["down2.xf.ff.proj.weight"] == (2 * 5120, 1280)
