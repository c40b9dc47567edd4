"""The tensor-core attention's work split, walked on the host with the kernel's own
schedule functions (``dfp_attention_schedule_check``; no GPU needed).

A cut query-tile pair is merged by the CTA holding its first KV tiles; the kernel
relies on that piece ending its CTA's range and on every other piece of the pair
starting one (so the merging CTA only ever waits for pieces that wait for nothing),
and on its publisher and flag warps predicting those pieces from the range ends.
"""
import numpy as np
import pytest

SYNC, DISPLACED, NAIVE, CROSS = 0, 1, 2, 3
CTAS = [148, 147, 132, 100, 64, 37, 7, 2, 1]


def _check(L, Lp, N, heads, mode, kv_len=0, images=1, ctas=148, p_lo=0, p_hi=0, budget=-1):
    from patch_diffusion_unet_b200 import dfp
    return dfp.LIB.dfp_attention_schedule_check(L, Lp, N, heads, mode, kv_len, images, ctas, p_lo, p_hi, budget)


# (L, Lp, N, heads) of the workloads: 64x64 / 128x128 / 240x240 maps, the stage's 20 heads,
# and the ragged shapes of the parity tests
SHAPES = [
    (4096, 1024, 4, 10), (16384, 2048, 8, 10), (57600, 7200, 8, 10), (4096, 512, 8, 20),
    (960, 320, 3, 2), (3200, 800, 4, 2), (256, 64, 4, 2), (600, 200, 3, 2), (512, 512, 1, 3),
]


@pytest.mark.parametrize("budget", [-1, 0], ids=["own-budget", "whole-rounds"])
@pytest.mark.parametrize("shape", SHAPES, ids=[f"L{s[0]}-N{s[2]}" for s in SHAPES])
@pytest.mark.parametrize("mode", [SYNC, DISPLACED, NAIVE], ids=["sync", "displaced", "naive"])
def test_self_attention_split(shape, mode, budget):
    """budget 0 deals whole units whenever there are at least as many units as CTAs (the
    large-map split); -1 takes the kernel's own choice (whole rounds at the 240 x 240 map)."""
    L, Lp, N, heads = shape
    for images in (1, 2):
        for ctas in CTAS:
            assert _check(L, Lp, N, heads, mode, images=images, ctas=ctas, budget=budget) == 0, (images, ctas)


@pytest.mark.parametrize("kv_len", [1, 77, 128, 129, 300])
@pytest.mark.parametrize("images", [1, 2, 3])
def test_cross_attention_split(images, kv_len):
    """The context's key count sets the one partial tile (none at 128)."""
    for ctas in CTAS:
        assert _check(4096, 4096, 1, 20, CROSS, kv_len=kv_len, images=images, ctas=ctas) == 0


def test_random_splits():
    rng = np.random.default_rng(7)
    for _ in range(300):
        N = int(rng.integers(1, 9))
        Lp = int(rng.integers(1, 80)) * 8
        heads = int(rng.integers(1, 12))
        mode = int(rng.integers(0, 3))
        images = int(rng.integers(1, 4))
        ctas = int(rng.integers(1, 200))
        for budget in (-1, 0):
            assert _check(N * Lp, Lp, N, heads, mode, images=images, ctas=ctas, budget=budget) == 0, \
                (N, Lp, heads, mode, images, ctas, budget)


@pytest.mark.parametrize("shape", SHAPES[:3], ids=["L4096", "L16384", "L57600"])
@pytest.mark.parametrize("world", [2, 4, 8])
def test_patch_range_split(shape, world):
    """A patch-parallel rank lists only its own query patches: every rank's range of the
    displaced step splits as cleanly as the whole list."""
    L, Lp, N, heads = shape
    if N % world:
        pytest.skip("patches do not divide among the ranks")
    per = N // world
    for r in range(world):
        for ctas in CTAS:
            for budget in (-1, 0):
                assert _check(L, Lp, N, heads, DISPLACED, ctas=ctas, p_lo=r * per, p_hi=(r + 1) * per,
                              budget=budget) == 0, (r, ctas, budget)


def test_bad_arguments():
    assert _check(4096, 1024, 4, 10, DISPLACED, p_lo=3, p_hi=3) == 1
    assert _check(4096, 1024, 4, 10, DISPLACED, p_lo=0, p_hi=5) == 1
    assert _check(0, 0, 1, 1, SYNC) == 1
    assert _check(4096, 1024, 4, 10, 9) == 1
    assert _check(4096, 1024, 4, 10, SYNC, ctas=0) == 1
