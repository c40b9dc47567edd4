"""Parity of the CUDA path (through the C ABI) against the CPU oracle, on a B200.

Every comparison is element by element on the same seeded inputs; the bar is
the relative L2 error of the whole compared tensor (1e-5 for fp32 storage, 2e-2
for bf16), per step, for the block output and for every intermediate stage.
Large workloads compare a sample of query tokens: the oracle computes all of
the state (GroupNorm statistics, conv, K/V) exactly and the attention output
only for the sampled rows.
"""
import numpy as np
import pytest
import torch

from patch_diffusion_unet_b200 import configs, inputs
from tests.parity_util import TOL, run_parity, worst

pytestmark = pytest.mark.gpu

STAGES = ("y", "y1", "h", "t", "q", "k", "v", "o")


def _assert(results, tol, stages=STAGES):
    for r in results:
        for s in stages:
            if s in r:
                assert r[s][0] <= tol, f"step {r['step']} stage {s}: rel-L2 {r[s][0]:.3e} > {tol} (max-abs {r[s][1]:.3e})"
        if "halo_ok" in r:
            assert r["halo_ok"], f"step {r['step']}: halo rows are not the expected copies"


def _sample(L, n, seed=1):
    rng = np.random.default_rng(seed)
    s = np.sort(rng.choice(L, size=min(n, L), replace=False))
    return np.unique(np.concatenate([s, [0, L - 1]]))


# ------------------------------------------------------------------ config 0 (fp32, SIMT)

@pytest.mark.parametrize("gn_mode,context", [(0, 0), (1, 0), (2, 0), (3, 0), (0, 1)],
                         ids=["corrected", "stale_others", "gn_sync", "gn_separate", "naive"])
def test_config0_fp32_all_steps(gn_mode, context):
    cfg = configs.get(0)
    res = run_parity(cfg, cfg["steps"], gn_mode=gn_mode, context=context)
    _assert(res, TOL["f32"])


def test_config0_fp32_random_affine_longer_run():
    cfg = configs.get(0, steps=8, n_sync=2)
    _assert(run_parity(cfg, 8, random_affine=True), TOL["f32"])


# ------------------------------------------------------------------ GroupNorm edge cases

def _jump_patch0(cfg, scale=10.0):
    """Step 0 with patch 0 scaled by `scale`, later steps unchanged: on step 1 (the first
    displaced step) the corrected estimate of patch 0's variance, avg_j V_j + (v_0 - V_0),
    is negative (the stale V_0 is scale^2 times the fresh v_0), so the clamp at 0 decides it."""
    R = cfg["H"] // cfg["n_patches"]

    def fn(t, x):
        if t != 0:
            return x
        x = np.array(x, copy=True)
        x[..., :R, :, :] = inputs.round_to(scale * x[..., :R, :, :], cfg["dtype"])
        return x
    return fn


@pytest.mark.parametrize("cfg", [configs.get(0), dict(configs.get(0), name="r40-bf16", H=24, W=40, C=128,
                                                      n_patches=3, gn_groups=8, heads=2, dtype="bf16",
                                                      steps=4, n_sync=1)],
                         ids=["fp32-16x16x64", "bf16-24x40x128"])
def test_groupnorm_variance_clamp(cfg):
    """A displaced step right after an input jump: the oracle clamps patch 0's GN1 variance
    (asserted here on the CPU side), and the GPU path matches it at every stage."""
    orc = []
    res = run_parity(cfg, cfg["steps"], x_fn=_jump_patch0(cfg), orc_out=orc)
    mu, var = orc[1]["gn1"]
    assert np.all(var[0] == 0.0), "the oracle did not clamp: the test input does not reach the clamp"
    assert np.all(var[1:] > 0.0)
    _assert(res, TOL[cfg["dtype"]])


def test_groupnorm_large_mean_fp32():
    """x + 30 (mean 30, spread about 1) at the fp32 bar: the statistics must not lose the
    variance to the cancellation of E[x^2] - E[x]^2 (at mean 30, E[x^2] ~ 901)."""
    cfg = configs.get(0)
    shift = lambda t, x: inputs.round_to(np.asarray(x, np.float64) + 30.0, "f32")  # noqa: E731
    _assert(run_parity(cfg, cfg["steps"], x_fn=shift), TOL["f32"])
    _assert(run_parity(cfg, cfg["steps"], x_fn=shift, gn_mode=1), TOL["f32"])


def test_groupnorm_large_mean_bf16_tcgen05():
    cfg = RAGGED_MEAN
    shift = lambda t, x: inputs.round_to(np.asarray(x, np.float64) + 30.0, "bf16")  # noqa: E731
    _assert(run_parity(cfg, cfg["steps"], x_fn=shift, random_affine=True), TOL["bf16"])


RAGGED_MEAN = dict(name="r40m", H=24, W=40, C=128, n_patches=3, gn_groups=8, gn_eps=1e-5, heads=2, head_dim=64,
                   dtype="bf16", block="res_attn", steps=5, n_sync=2)


# ------------------------------------------------------------------ small bf16 shapes (ragged tiles)

RAGGED = [
    # W < 128, 128 % W != 0, patch token count not a multiple of 128 (conv tiles 2 rows x 40 cols)
    dict(name="r40", H=24, W=40, C=128, n_patches=3, gn_groups=8, gn_eps=1e-5, heads=2, head_dim=64,
         dtype="bf16", block="res_attn", steps=5, n_sync=2),
    # W > 128: two column tiles per row, the second one partly outside the map
    dict(name="r200", H=16, W=200, C=128, n_patches=4, gn_groups=8, gn_eps=1e-5, heads=2, head_dim=64,
         dtype="bf16", block="res_attn", steps=5, n_sync=2),
    # one row per patch: a row is both the first and the last of its patch
    dict(name="r1", H=4, W=64, C=128, n_patches=4, gn_groups=8, gn_eps=1e-5, heads=2, head_dim=64,
         dtype="bf16", block="res_attn", steps=5, n_sync=2),
    # an odd number of conv tiles (3 patches x 5 one-row tiles): the last CTA pair of the
    # conv GEMM has a padding tile (zero-filled loads, no stores)
    dict(name="r15", H=15, W=40, C=128, n_patches=3, gn_groups=8, gn_eps=1e-5, heads=2, head_dim=64,
         dtype="bf16", block="res_attn", steps=5, n_sync=2),
    # N = 1 (no cross-patch context at all)
    dict(name="n1", H=16, W=32, C=192, n_patches=1, gn_groups=8, gn_eps=1e-5, heads=3, head_dim=64,
         dtype="bf16", block="res_attn", steps=4, n_sync=1),
]


@pytest.mark.parametrize("cfg", RAGGED, ids=[c["name"] for c in RAGGED])
@pytest.mark.parametrize("family", [0, 1], ids=["tcgen05", "simt"])
def test_ragged_bf16(cfg, family):
    _assert(run_parity(cfg, cfg["steps"], family=family, random_affine=True), TOL["bf16"])


def test_peaked_attention_bf16():
    """Large q/k weights make the softmax peaked, stressing the running maximum."""
    cfg = RAGGED[0]
    scale = {"attn.to_q.weight": 12.0, "attn.to_k.weight": 12.0}
    _assert(run_parity(cfg, cfg["steps"], weight_scale=scale), TOL["bf16"])


@pytest.mark.parametrize("gn_mode,context", [(1, 0), (2, 0), (3, 0), (0, 1)],
                         ids=["stale_others", "gn_sync", "gn_separate", "naive"])
@pytest.mark.parametrize("family", [0, 1], ids=["tcgen05", "simt"])
def test_modes_bf16(gn_mode, context, family):
    cfg = RAGGED[1]
    _assert(run_parity(cfg, cfg["steps"], gn_mode=gn_mode, context=context, family=family), TOL["bf16"])


# ------------------------------------------------------------------ configs 1-3 (full sizes)

def test_config1_first_steps_all_stages():
    cfg = configs.get(1)
    _assert(run_parity(cfg, 8), TOL["bf16"])


def test_config1_whole_unit_rounds():
    """The attention's large-map split forced onto config 1 (a K/V budget of one byte): one
    round of whole (head, patch, pair) units dealt one per CTA, then the 12 remaining units
    split stream-K, each CTA's first tail piece first and its merging piece last."""
    cfg = configs.get(1)
    _assert(run_parity(cfg, 5, kv_budget=1), TOL["bf16"])


def test_config1_simt_cross_check():
    cfg = configs.get(1)
    _assert(run_parity(cfg, 7, family=1), TOL["bf16"])


def test_config1_full_run_sampled_tokens():
    cfg = configs.get(1)
    L = cfg["H"] * cfg["W"]
    res = run_parity(cfg, cfg["steps"], query_tokens=_sample(L, 256), stages=False)
    _assert(res, TOL["bf16"], stages=("y",))


def test_config2_sampled_tokens():
    cfg = configs.get(2)
    L = cfg["H"] * cfg["W"]
    _assert(run_parity(cfg, 7, query_tokens=_sample(L, 384)), TOL["bf16"])


def test_config3_steps_1_2_sampled_tokens():
    """The 240x240 map, compared on steps 1 (sync) and 2 (first displaced step)."""
    cfg = configs.get(3)
    L = cfg["H"] * cfg["W"]
    # sample around every patch boundary plus random tokens
    Lp = L // cfg["n_patches"]
    edges = np.concatenate([[p * Lp - 1, p * Lp, p * Lp + 127, p * Lp + 128] for p in range(1, cfg["n_patches"])])
    tok = np.unique(np.concatenate([_sample(L, 256), edges]))
    res = run_parity(cfg, 3, oracle_from=1, query_tokens=tok)
    assert [r["step"] for r in res] == [1, 2]
    _assert(res, TOL["bf16"])


# ------------------------------------------------------------------ behaviour

def test_deterministic_bitwise():
    from patch_diffusion_unet_b200 import dfp
    cfg = configs.get(1)
    outs = []
    for _ in range(2):
        wl = inputs.SyntheticWorkload(cfg)
        blk = dfp.DisplacedPatchBlock(cfg)
        blk.load_weights(wl.weights)
        for t, s in wl.schedule()[:7]:
            blk.step(inputs.to_torch(wl.x(t), "bf16").cuda(), t, s)
        outs.append(blk.output().clone())
        blk.check_device()
        blk.close()
    assert torch.equal(outs[0], outs[1])


def test_state_errors_on_gpu():
    from patch_diffusion_unet_b200 import dfp
    cfg = configs.get(0)
    wl = inputs.SyntheticWorkload(cfg)
    blk = dfp.DisplacedPatchBlock(cfg)
    x = inputs.to_torch(wl.x(0), "f32").cuda()
    with pytest.raises(dfp.DfpError) as e:
        blk.step(x, 0, 1)                      # weights missing
    assert e.value.status == dfp.E_STATE
    blk.load_weights(wl.weights)
    with pytest.raises(dfp.DfpError) as e:
        blk.step(x, 0, 0)                      # step 0 must be synchronous
    assert e.value.status == dfp.E_STATE
    blk.step(x, 0, 1)
    with pytest.raises(dfp.DfpError) as e:
        blk.step(x, 2, 0)                      # steps must be consecutive
    assert e.value.status == dfp.E_STATE
    with pytest.raises(dfp.DfpError) as e:
        blk.set_kernel_family(0)               # no tensor-core path for fp32
    assert e.value.status == dfp.E_UNSUPPORTED
    blk.step(x, 1, 0)
    blk.check_device()
    blk.close()


def test_host_buffer_step_matches_device_step():
    from patch_diffusion_unet_b200 import dfp
    cfg = configs.get(1)
    wl = inputs.SyntheticWorkload(cfg)
    a, b = dfp.DisplacedPatchBlock(cfg), dfp.DisplacedPatchBlock(cfg)
    a.load_weights(wl.weights)
    b.load_weights(wl.weights)
    y_host = torch.empty(cfg["H"] * cfg["W"], cfg["C"], dtype=torch.bfloat16).pin_memory()
    for t, s in wl.schedule()[:7]:
        xh = inputs.to_torch(wl.x(t), "bf16").pin_memory()
        a.step(xh.cuda(), t, s)
        b.step_host(xh, y_host, t, s)
        assert torch.equal(a.output().cpu(), y_host)
    a.close()
    b.close()


@pytest.mark.gpu
@pytest.mark.parametrize("cfg_id", [1, 4])
def test_pipelined_host_steps_match_device_steps(cfg_id):
    """dfp_step_host_async: consecutive calls without waiting (copies overlapped with the
    neighbouring steps), then one synchronize; every step's output equals the device path's."""
    from patch_diffusion_unet_b200 import dfp
    cfg = configs.get(cfg_id)
    wl = inputs.SyntheticWorkload(cfg)
    weights = dict(wl.weights, context=wl.context) if wl.context is not None else wl.weights
    a, b = dfp.DisplacedPatchBlock(cfg), dfp.DisplacedPatchBlock(cfg)
    a.load_weights(weights)
    b.load_weights(weights)
    sched = wl.schedule()[:8]
    xs = [inputs.to_torch(wl.x(t), "bf16").pin_memory() for t, _ in sched]
    ys = [torch.empty(cfg["H"] * cfg["W"], cfg["C"], dtype=torch.bfloat16).pin_memory() for _ in sched]
    for i, (t, s) in enumerate(sched):
        b.step_host_async(xs[i], ys[i], t, s)
    b.synchronize()
    for i, (t, s) in enumerate(sched):
        a.step(xs[i].cuda(), t, s)
        assert torch.equal(a.output().cpu(), ys[i]), f"step {t}"
    a.close()
    b.close()
