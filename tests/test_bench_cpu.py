"""The benchmark's accounting on the CPU: the algorithmic work per launch that the roofline
divides by the measured time, and the guard on the recorded DRAM traffic.

The expected FLOP counts are the closed forms of each contraction (2 FLOP per
multiply-add; attention 4 L^2 d heads, two GEMMs per score), evaluated by hand for
the named workloads: e.g. the 64x64x640 conv is 2 * 4096 * 640 * 9 * 640 = 30.2 GFLOP.
"""
import pytest

import bench
from patch_diffusion_unet_b200 import configs

GF = 1e9


@pytest.mark.parametrize("cid,conv,qkv,attn,out,total", [
    (1, 30.1990, 10.0663, 42.9497, 3.35544, 86.5704),
    (2, 120.796, 40.2653, 687.195, 13.4218, 861.678),
    (3, 424.673, 141.558, 8493.47, 47.1859, 9106.88),
])
def test_res_attn_work_per_launch(cid, conv, qkv, attn, out, total):
    wm = bench.work_model(configs.get(cid))
    assert wm["conv (tcgen05)"] == ("tensor", pytest.approx(conv * GF, rel=1e-4))
    assert wm["qkv (tcgen05)"] == ("tensor", pytest.approx(qkv * GF, rel=1e-4))
    assert wm["attention (tcgen05)"] == ("tensor", pytest.approx(attn * GF, rel=1e-4))
    assert wm["out projection (tcgen05)"] == ("tensor", pytest.approx(out * GF, rel=1e-4))
    assert wm["_total_flops"] == pytest.approx(total * GF, rel=1e-4)


def test_groupnorm_bytes_per_launch():
    """GN1 reads and writes the map once and copies 2 halo rows per inner patch boundary in
    each direction; GN2 reads and writes the map once (bf16: 2 bytes)."""
    cfg = configs.get(1)
    L, C, W, N = 64 * 64, 640, 64, 4
    wm = bench.work_model(cfg)
    assert wm["gn2 (fused)"] == ("hbm", 2 * L * C * 2)
    assert wm["gn1 + SiLU + halo (fused)"] == ("hbm", 2 * L * C * 2 + 2 * 2 * (N - 1) * W * C * 2)


def test_stage_work_per_step():
    """64x64x1280 stage, two transformer blocks: 899.8 GFLOP per step (the context K/V
    projection, 1.6 GFLOP, runs once when the weights are loaded, not per step)."""
    wm = bench.work_model(configs.get(4))
    L, C, F, T, heads = 4096, 1280, 5120, 77, 20
    assert wm["conv1 (tcgen05)"][1] == pytest.approx(2.0 * L * C * 9 * C)
    assert wm["self-attention (tcgen05)"][1] == pytest.approx(4.0 * L * L * 64 * heads)
    assert wm["cross-attention (tcgen05)"][1] == pytest.approx(4.0 * L * T * 64 * heads)
    assert wm["ff proj + GEGLU (tcgen05)"][1] == pytest.approx(2.0 * L * C * 2 * F)
    assert wm["_total_flops"] == pytest.approx(899.8 * GF, rel=2e-4)


def test_batch_scales_every_launch():
    one, two = bench.work_model(configs.get(1)), bench.work_model(configs.get(1, batch=2))
    for k, v in one.items():
        if isinstance(v, tuple):
            assert two[k] == (v[0], 2 * v[1])
    assert two["_total_flops"] == 2 * one["_total_flops"]
    assert two["_rows_per_patch"] == one["_rows_per_patch"]


def test_traffic_only_for_the_captured_source(monkeypatch):
    """A recorded ncu traffic figure applies only while the kernel's sources hash the same."""
    import hashlib
    import os
    files = ("tc_attention.cu", "dfp_common.cuh", "exp2_poly.cuh")
    m = hashlib.sha256()
    for fn in files:
        with open(os.path.join(bench.ROOT, "patch_diffusion_unet_b200", "csrc", fn), "rb") as f:
            m.update(f.read())
    key = ("some-workload", "attention (tcgen05)")
    monkeypatch.setitem(bench.NCU_TRAFFIC, key, (123.0e6, files, m.hexdigest()[:16]))
    assert bench.ncu_traffic(*key) == 123.0e6
    assert bench.ncu_traffic("some-other-workload", "attention (tcgen05)") is None
    monkeypatch.setitem(bench.NCU_TRAFFIC, key, (123.0e6, files, "0" * 16))
    assert bench.ncu_traffic(*key) is None
