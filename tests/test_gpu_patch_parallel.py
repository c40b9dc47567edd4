"""Patch parallelism on a B200, with the ranks emulated in one process: every rank is its
own library handle computing its patch range (dfp_step_patches) on displaced steps and the
whole map on synchronous ones; the exchange between steps is the product's, over the
one-process transport (copies between the handles' buffers; no kernel of one rank waits on
another's).  Every rank's assembled output is compared with the CPU oracle's single-device
displaced step at every step."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from patch_diffusion_unet_b200 import configs, inputs
from tests.parity_util import TOL, host, rel_l2

pytestmark = pytest.mark.gpu

SMALL = dict(name="pp-r40", H=32, W=40, C=128, n_patches=4, gn_groups=8, gn_eps=1e-5, heads=2, head_dim=64,
             dtype="bf16", block="res_attn", steps=6, n_sync=2)


def _run(cfg, world, n_steps, oracle_from=0, query_tokens=None, gn_mode=0):
    from patch_diffusion_unet_b200 import patch_parallel as pp
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    stream = torch.cuda.current_stream()
    ranks = [pp.PatchParallelLayer(cfg, r, world, stream=stream, gn_mode=gn_mode) for r in range(world)]
    for L in ranks:
        L.load_weights(wl.weights)
    orc = oracle.make_block(cfg, wl.weights, gn_mode=["corrected", "stale_others", "sync", "separate"][gn_mode])
    transport = pp.LocalTransport()
    errs = []
    for t, is_sync in wl.schedule()[:n_steps]:
        x = wl.x(t)
        xd = inputs.to_torch(x, cfg["dtype"]).cuda()
        for L in ranks:
            L.compute(xd, t, is_sync)
        pp.exchange(ranks, transport, t, is_sync)
        torch.cuda.synchronize()
        for L in ranks:
            L.blk.check_device()
        if t < oracle_from:
            continue
        want = orc.step(x, t - oracle_from, is_sync, query_tokens=query_tokens)["y"]
        y0 = host(ranks[0].output())
        for L in ranks[1:]:
            assert np.array_equal(host(L.output()), y0), f"step {t}: rank {L.rank} holds another output"
        got = y0 if query_tokens is None else y0[query_tokens]
        errs.append((t, is_sync, rel_l2(got, want)))
    for L in ranks:
        L.close()
    return errs


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("gn_mode", [0, 1, 3], ids=["corrected", "stale_others", "gn_separate"])
def test_small_map_all_steps(world, gn_mode):
    errs = _run(SMALL, world, SMALL["steps"], gn_mode=gn_mode)
    assert sum(1 for e in errs if not e[1]) >= 4
    assert max(e[2] for e in errs) <= TOL["bf16"], errs


@pytest.mark.parametrize("world", [2, 4])
def test_config1_first_steps(world):
    cfg = configs.get(1)
    errs = _run(cfg, world, 9)
    assert max(e[2] for e in errs) <= TOL["bf16"], errs


def test_config3_two_ranks_first_displaced_steps():
    """The 240x240 map over two ranks: steps 1 (sync) to 3 (two displaced steps), sampled
    query tokens around every patch edge."""
    cfg = configs.get(3)
    L = cfg["H"] * cfg["W"]
    Lp = L // cfg["n_patches"]
    rng = np.random.default_rng(5)
    edges = np.concatenate([[p * Lp - 1, p * Lp, p * Lp + 127] for p in range(1, cfg["n_patches"])])
    tok = np.unique(np.concatenate([rng.choice(L, 192, replace=False), edges, [0, L - 1]]))
    errs = _run(cfg, 2, 4, oracle_from=1, query_tokens=tok)
    assert [e[0] for e in errs] == [1, 2, 3]
    assert max(e[2] for e in errs) <= TOL["bf16"], errs


def test_range_step_argument_and_state_checks():
    from patch_diffusion_unet_b200 import dfp
    cfg = SMALL
    wl = inputs.SyntheticWorkload(cfg)
    blk = dfp.DisplacedPatchBlock(cfg)
    blk.load_weights(wl.weights)
    x = inputs.to_torch(wl.x(0), "bf16").cuda()
    p = ctypes.c_void_p(x.data_ptr())
    assert dfp.LIB.dfp_step_patches(blk.h, p, 0, 0, 2) == dfp.E_STATE      # step 0 must be synchronous
    blk.step(x, 0, 1)
    assert dfp.LIB.dfp_step_patches(blk.h, p, 1, 2, 2) == dfp.E_ARG        # empty range
    assert dfp.LIB.dfp_step_patches(blk.h, p, 1, 0, 5) == dfp.E_ARG        # past the last patch
    assert dfp.LIB.dfp_step_patches(blk.h, p, 2, 0, 2) == dfp.E_STATE      # not the next step
    assert dfp.LIB.dfp_step_patches(blk.h, p, 1, 0, 2) == dfp.OK
    blk.check_device()
    blk.close()
    for over, gn in ((dict(dtype="f32"), 0), ({}, 2)):
        c = dict(cfg, **over)
        w = inputs.SyntheticWorkload(c)
        b = dfp.DisplacedPatchBlock(c, gn_mode=gn)
        b.load_weights(w.weights)
        xx = inputs.to_torch(w.x(0), c["dtype"]).cuda()
        b.step(xx, 0, 1)
        assert dfp.LIB.dfp_step_patches(b.h, ctypes.c_void_p(xx.data_ptr()), 1, 0, 2) == dfp.E_UNSUPPORTED
        b.close()
