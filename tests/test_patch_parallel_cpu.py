"""Patch parallelism across ranks, on the host: the partition, the layout of the
all-gathers, and whole runs of gloo ranks (127.0.0.1) whose exchange is the product's
(patch_diffusion_unet_b200.patch_parallel) and whose per-rank compute is the oracle-based
stand-in of tests/patch_parallel_ref.py; every rank's assembled output must equal the
single-process oracle at every step, synchronous and displaced."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from patch_diffusion_unet_b200 import patch_parallel as pp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CFG = dict(name="pp-small", H=16, W=6, C=64, n_patches=4, gn_groups=8, gn_eps=1e-5, heads=1, head_dim=64,
           dtype="f32", block="res_attn", steps=6, n_sync=2)


def test_partition():
    assert [pp.partition(8, 4, r) for r in range(4)] == [(0, 2), (2, 4), (4, 6), (6, 8)]
    assert pp.partition(8, 1, 0) == (0, 8)
    with pytest.raises(ValueError):
        pp.partition(6, 4, 0)
    with pytest.raises(ValueError):
        pp.partition(8, 2, 2)


@pytest.mark.parametrize("world", [1, 2, 4])
def test_gathers_cover_every_buffer_once(world):
    """The ranks' own chunks tile each gathered buffer exactly: no byte missed or doubled."""
    cfg = dict(CFG, heads=2, C=128, dtype="bf16")
    e, Lp, R = pp.layout(cfg)
    sizes = {"k": 2 * cfg["H"] * cfg["W"] * 64 * e, "v": 2 * cfg["H"] * cfg["W"] * 64 * e,
             "mom1": cfg["n_patches"] * cfg["gn_groups"] * 8, "mom2": cfg["n_patches"] * cfg["gn_groups"] * 8,
             "y": cfg["H"] * cfg["W"] * cfg["C"] * e}
    bufs = {k: torch.zeros(n, dtype=torch.uint8) for k, n in sizes.items()}
    for r in range(world):
        for full, own in pp.gathers(cfg, lambda n, par: bufs[n], 0, r, world):
            assert full.numel() == world * own.numel()
            own += 1
    for k, b in bufs.items():
        assert torch.all(b == 1), k


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, gn_mode, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import oracle
    from patch_diffusion_unet_b200 import inputs
    from patch_diffusion_unet_b200 import patch_parallel as ppm
    from tests.patch_parallel_ref import OracleRank
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = inputs.SyntheticWorkload(CFG, random_affine=True)
        layer = OracleRank(CFG, wl.weights, rank, world, gn_mode=gn_mode)
        ref = oracle.make_block(CFG, wl.weights, gn_mode=gn_mode)
        transport = ppm.DistTransport()
        errs = []
        for t, is_sync in wl.schedule():
            x = wl.x(t)
            layer.compute(x, t, is_sync)
            ppm.exchange([layer], transport, t, is_sync)
            want = ref.step(x, t, is_sync)["y"]
            got = layer.output()
            errs.append(float(np.linalg.norm(got - want) / np.linalg.norm(want)))
        out[rank] = errs
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world,gn_mode", [(2, "corrected"), (4, "corrected"), (2, "stale_others"),
                                           (2, "separate")])
def test_ranks_reproduce_the_single_process_oracle(world, gn_mode):
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, gn_mode, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(200)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for r in range(world):
        errs = out[r]
        assert len(errs) == CFG["steps"]
        assert max(errs) <= 1e-5, (r, errs)


def test_displaced_without_exchange_is_wrong():
    """Negative control: skipping the exchange leaves the other patches' context one step
    too old on the second displaced step, and the output moves away from the oracle."""
    import oracle
    from patch_diffusion_unet_b200 import inputs
    from tests.patch_parallel_ref import OracleRank
    wl = inputs.SyntheticWorkload(CFG, random_affine=True)
    world = 2
    ranks = [OracleRank(CFG, wl.weights, r, world) for r in range(world)]
    ref = oracle.make_block(CFG, wl.weights)
    worst = 0.0
    for t, is_sync in wl.schedule():
        x = wl.x(t)
        for L in ranks:
            L.compute(x, t, is_sync)
        if is_sync:
            pp.exchange(ranks, pp.LocalTransport(), t, is_sync)    # halo rows only
        want = ref.step(x, t, is_sync)["y"]
        got = ranks[0].output()
        R = CFG["H"] // CFG["n_patches"] * CFG["W"]
        p0, p1 = ranks[0].p0, ranks[0].p1
        worst = max(worst, float(np.linalg.norm(got[p0 * R:p1 * R] - want[p0 * R:p1 * R]) /
                                 np.linalg.norm(want[p0 * R:p1 * R])))
    assert worst > 1e-4


def test_local_transport_matches_gloo_layout():
    """The one-process transport reproduces the oracle too (the GPU test's transport)."""
    import oracle
    from patch_diffusion_unet_b200 import inputs
    from tests.patch_parallel_ref import OracleRank
    wl = inputs.SyntheticWorkload(CFG, random_affine=True)
    world = 4
    ranks = [OracleRank(CFG, wl.weights, r, world) for r in range(world)]
    ref = oracle.make_block(CFG, wl.weights)
    for t, is_sync in wl.schedule():
        x = wl.x(t)
        for L in ranks:
            L.compute(x, t, is_sync)
        pp.exchange(ranks, pp.LocalTransport(), t, is_sync)
        want = ref.step(x, t, is_sync)["y"]
        for L in ranks:
            got = L.output()
            assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 1e-5, (t, L.rank)
