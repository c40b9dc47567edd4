"""Pins of the CPU oracle against things other than itself (CPU only).

* synchronous steps, N=1 steps and steps whose stale context equals the fresh
  one must reproduce the single-device layer ("DistriFusion" project README,
  Overview (a) vs (c): the method changes only where context comes from), which
  is written with PyTorch's fp64 library routines in ``torch_ref``;
* the naive-patch baseline (README Overview (b)) must equal the single-device
  layer run on each patch alone;
* a hand-worked GroupNorm example (``golden/gn_corrected_hand_example.json``);
* brute-force loops on tiny inputs for every displaced layer;
* locality of the conv halo and the exact K/V set of displaced attention.
"""
import copy
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from patch_diffusion_unet_b200 import configs, inputs
from tests import torch_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

SMALL = dict(name="small", H=8, W=6, C=32, n_patches=4, gn_groups=4, gn_eps=1e-5, heads=4,
             head_dim=8, dtype="f32", block="res_attn", steps=4, n_sync=1)
STAGE = dict(name="stage-small", H=8, W=4, C=32, n_patches=2, gn_groups=4, gn_eps=1e-5, heads=2,
             head_dim=16, dtype="f32", block="sdxl_stage", steps=3, n_sync=1, n_xformer=2,
             ffn_inner=48, ctx_len=5, ctx_dim=12)


def _close(a, b, tol=1e-10):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape, (a.shape, b.shape)
    err = np.abs(a - b).max()
    scale = max(np.abs(b).max(), 1e-30)
    assert err <= tol * scale, f"max-abs {err} vs scale {scale}"


def _block(cfg, wl, **kw):
    return oracle.make_block(cfg, wl.weights, wl.context, **kw)


def _full(cfg, x, wl):
    if cfg["block"] == "res_attn":
        return torch_ref.res_attn_full(x, wl.weights, cfg)
    return torch_ref.sdxl_stage_full(x, wl.weights, wl.context, cfg)


# --------------------------------------------------------------------------- golden

def test_gn_hand_example_merge():
    g = json.load(open(os.path.join(GOLDEN, "gn_corrected_hand_example.json")))
    st = lambda v: [np.mean(v), np.mean(np.square(v))]
    stale = np.array([[st(g["patch0_stale_values"])], [st(g["patch1_stale_values"])]])
    fresh = np.array([[st(g["patch0_fresh_values"])], [st(g["patch1_fresh_values"])]])
    for mode in ("corrected", "stale_others"):
        mu, var = oracle.merge_moments(fresh, stale, False, mode)
        exp = g["expected"][mode]
        assert mu[0, 0] == pytest.approx(exp["mu"], abs=1e-12)
        assert var[0, 0] == pytest.approx(exp["var"], abs=1e-12)
        assert mu[0, 0] ** 2 + var[0, 0] == pytest.approx(exp["E2"], abs=1e-12)


def test_gn_hand_example_through_layer():
    """Same example through the stateful layer: a step at t-1, then a displaced step at t."""
    g = json.load(open(os.path.join(GOLDEN, "gn_corrected_hand_example.json")))
    prev = np.array(g["patch0_stale_values"] + g["patch1_stale_values"]).reshape(2, 2, 1)
    cur = np.array(g["patch0_fresh_values"] + g["patch1_fresh_values"]).reshape(2, 2, 1)
    for mode in ("corrected", "stale_others"):
        gn = oracle.DisplacedGroupNorm(2, 1, 0.0, np.ones(1), np.zeros(1), mode)
        gn(prev, is_sync=True)
        out = gn(cur, is_sync=False)
        exp = g["expected"][mode]
        assert gn.last[0][0, 0] == pytest.approx(exp["mu"])
        assert gn.last[1][0, 0] == pytest.approx(exp["var"])
        _close(out[0, :, 0], (np.array(g["patch0_fresh_values"]) - exp["mu"]) / math.sqrt(exp["var"]))


def test_gn_clamp_hand_example():
    """A displaced step whose corrected variance estimate is negative: the oracle clamps it
    to 0, so patch 0 is normalised by 1/sqrt(eps) (eps = 1/4 here: outputs are x * 2)."""
    g = json.load(open(os.path.join(GOLDEN, "gn_clamp_hand_example.json")))
    prev = np.array(g["patch0_stale_values"] + g["patch1_stale_values"]).reshape(2, 2, 1)
    cur = np.array(g["patch0_fresh_values"] + g["patch1_fresh_values"]).reshape(2, 2, 1)
    for mode in ("corrected", "stale_others"):
        gn = oracle.DisplacedGroupNorm(2, 1, g["eps"], np.ones(1), np.zeros(1), mode)
        gn(prev, is_sync=True)
        out = gn(cur, is_sync=False)
        exp = g["expected"][mode]
        assert gn.last[0][0, 0] == pytest.approx(exp["mu"], abs=1e-12)
        assert gn.last[1][0, 0] == exp["var"]
        _close(out[0, :, 0], np.array(exp["patch0_out"]))


# --------------------------------------------------------------------------- library pins

@pytest.mark.parametrize("cfg", [configs.get(0), SMALL, configs.get(SMALL, n_patches=2),
                                 configs.get(SMALL, n_patches=1)], ids=["cfg0", "n4", "n2", "n1"])
def test_sync_step_equals_full_layer(cfg):
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    blk = _block(cfg, wl)
    x = wl.x(0)
    out = blk.step(x, 0, 1)
    ref = _full(cfg, x.astype(np.float64), wl)
    for k in ("y1", "h", "t"):
        _close(out[k], ref[k])
    _close(out["o"], ref["o"])
    _close(out["y"], ref["y"])


def test_n1_displaced_equals_full_layer():
    cfg = configs.get(SMALL, n_patches=1)
    wl = inputs.SyntheticWorkload(cfg)
    blk = _block(cfg, wl)
    for t in range(4):
        x = wl.x(t)
        _close(blk.step(x, t, int(t == 0))["y"], _full(cfg, x.astype(np.float64), wl)["y"])


@pytest.mark.parametrize("mode", ["corrected", "stale_others"])
@pytest.mark.parametrize("N", [2, 4])
def test_stale_equal_to_fresh_gives_full_layer(mode, N):
    cfg = configs.get(SMALL, n_patches=N)
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    blk = _block(cfg, wl, gn_mode=mode)
    x = wl.x(0)
    blk.step(x, 0, 1)
    out = blk.step(x, 1, 0)          # displaced, but the cache holds this very map
    ref = _full(cfg, x.astype(np.float64), wl)
    _close(out["y"], ref["y"])
    _close(out["t"], ref["t"])


def test_displaced_differs_from_sync():
    """Sanity: with a drifting input a displaced step is not the full layer."""
    cfg = SMALL
    wl = inputs.SyntheticWorkload(cfg)
    blk = _block(cfg, wl)
    blk.step(wl.x(0), 0, 1)
    x1 = wl.x(1)
    y = blk.step(x1, 1, 0)["y"]
    ref = _full(cfg, x1.astype(np.float64), wl)["y"]
    assert np.abs(y - ref).max() > 1e-6


def test_naive_context_equals_independent_patches():
    cfg = SMALL
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    blk = _block(cfg, wl, context="naive")
    blk.step(wl.x(0), 0, 1)
    x = wl.x(1)
    y = blk.step(x, 1, 0)["y"].reshape(cfg["H"], cfg["W"], cfg["C"])
    R = cfg["H"] // cfg["n_patches"]
    for p in range(cfg["n_patches"]):
        part = x[p * R:(p + 1) * R].astype(np.float64)
        ref = torch_ref.res_attn_full(part, wl.weights, configs.get(cfg, H=R))["y"]
        _close(y[p * R:(p + 1) * R].reshape(-1, cfg["C"]), ref)


# --------------------------------------------------------------------------- GroupNorm-only modes (R8)

def _gn_lib(x, G, gamma, beta, eps, silu):
    """PyTorch's group_norm (+ SiLU) on one [rows, W, C] map, fp64."""
    X = torch_ref._nchw(x)
    y = torch.nn.functional.group_norm(X, G, torch_ref._t(gamma), torch_ref._t(beta), eps)
    return torch_ref._nhwc(torch.nn.functional.silu(y) if silu else y)


@pytest.mark.parametrize("N", [2, 4])
def test_gn_sync_mode_displaced_step_normalises_with_the_full_map(N):
    """GroupNorm 'sync' mode: on a displaced step both GroupNorms equal PyTorch's group_norm
    over the whole map of this step, while the conv and the attention stay displaced
    (the output differs from the full layer)."""
    cfg = configs.get(SMALL, n_patches=N)
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    w = wl.weights
    blk = _block(cfg, wl, gn_mode="sync")
    blk.step(wl.x(0), 0, 1)
    x = wl.x(1).astype(np.float64)
    out = blk.step(x, 1, 0)
    G, eps = cfg["gn_groups"], cfg["gn_eps"]
    _close(out["y1"], _gn_lib(x, G, w["gn1.weight"], w["gn1.bias"], eps, True))
    _close(out["t"], _gn_lib(out["h"], G, w["gn2.weight"], w["gn2.bias"], eps, False))
    assert np.abs(out["y"] - _full(cfg, x, wl)["y"]).max() > 1e-6


@pytest.mark.parametrize("N", [2, 4])
def test_gn_separate_mode_displaced_step_normalises_each_patch_alone(N):
    """GroupNorm 'separate' mode: on a displaced step each patch's GroupNorm equals
    PyTorch's group_norm of that patch alone; the synchronous step stays the full layer."""
    cfg = configs.get(SMALL, n_patches=N)
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    w = wl.weights
    blk = _block(cfg, wl, gn_mode="separate")
    x0 = wl.x(0).astype(np.float64)
    _close(blk.step(x0, 0, 1)["y"], _full(cfg, x0, wl)["y"])
    x = wl.x(1).astype(np.float64)
    out = blk.step(x, 1, 0)
    G, eps, R = cfg["gn_groups"], cfg["gn_eps"], cfg["H"] // N
    for p in range(N):
        rows = slice(p * R, (p + 1) * R)
        _close(out["y1"][rows], _gn_lib(x[rows], G, w["gn1.weight"], w["gn1.bias"], eps, True))
        _close(out["t"][rows], _gn_lib(out["h"][rows], G, w["gn2.weight"], w["gn2.bias"], eps, False))


@pytest.mark.parametrize("mode", ["sync", "separate"])
def test_gn_modes_n1_and_stale_equal_fresh_give_full_layer(mode):
    """N = 1 at every step, and a displaced step whose cache holds this very map (sync
    mode), reproduce the full layer."""
    cfg = configs.get(SMALL, n_patches=1)
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    blk = _block(cfg, wl, gn_mode=mode)
    for t in range(3):
        x = wl.x(t).astype(np.float64)
        _close(blk.step(x, t, int(t == 0))["y"], _full(cfg, x, wl)["y"])
    if mode == "sync":
        cfg = configs.get(SMALL, n_patches=4)
        wl = inputs.SyntheticWorkload(cfg, random_affine=True)
        blk = _block(cfg, wl, gn_mode=mode)
        x = wl.x(0).astype(np.float64)
        blk.step(x, 0, 1)
        _close(blk.step(x, 1, 0)["y"], _full(cfg, x, wl)["y"])


# --------------------------------------------------------------------------- layer-level pins

def test_conv_halo_locality():
    rng = np.random.default_rng(3)
    N, H, W, C = 4, 16, 5, 3
    R = H // N
    conv = oracle.DisplacedConv3x3(N, rng.standard_normal((C, C, 3, 3)), rng.standard_normal(C))
    conv(rng.standard_normal((H, W, C)), True)
    prev = conv.prev.copy()
    y = rng.standard_normal((H, W, C))
    base = oracle.DisplacedConv3x3(N, conv.weight, conv.bias)
    base.prev = prev
    out0 = base(y, False)

    def run(prev2):
        c = oracle.DisplacedConv3x3(N, conv.weight, conv.bias)
        c.prev = prev2
        return c(y, False)

    j = 1
    for interior in (j * R + 1, j * R + 2):
        p2 = prev.copy()
        p2[interior] += 10.0
        _close(run(p2), out0, tol=0)
    # last row of patch j feeds only the first output row of patch j+1
    p2 = prev.copy()
    p2[(j + 1) * R - 1] += 10.0
    diff = np.abs(run(p2) - out0).max(axis=(1, 2))
    assert set(np.nonzero(diff)[0]) == {(j + 1) * R}
    # first row of patch j feeds only the last output row of patch j-1
    p2 = prev.copy()
    p2[j * R] += 10.0
    diff = np.abs(run(p2) - out0).max(axis=(1, 2))
    assert set(np.nonzero(diff)[0]) == {j * R - 1}


def test_conv_matches_conv2d_on_assembled_band():
    rng = np.random.default_rng(4)
    N, H, W, C, Co = 3, 9, 4, 2, 5
    R = H // N
    w, b = rng.standard_normal((Co, C, 3, 3)), rng.standard_normal(Co)
    prev = rng.standard_normal((H, W, C))
    y = rng.standard_normal((H, W, C))
    conv2 = oracle.DisplacedConv3x3(N, w, b)
    conv2.prev = prev
    out = conv2(y, False)
    for p in range(N):
        r0, r1 = p * R, (p + 1) * R
        top = prev[r0 - 1:r0] if p > 0 else np.zeros((1, W, C))
        bot = prev[r1:r1 + 1] if p < N - 1 else np.zeros((1, W, C))
        band = np.concatenate([top, y[r0:r1], bot])
        ref = F.conv2d(torch.from_numpy(band).permute(2, 0, 1)[None], torch.from_numpy(w),
                       torch.from_numpy(b), padding=(0, 1))[0].permute(1, 2, 0).numpy()
        _close(out[r0:r1], ref)


def test_displaced_attention_matches_sdpa_on_assembled_kv():
    rng = np.random.default_rng(5)
    N, Hh, W, C, heads = 3, 6, 4, 8, 2
    d = C // heads
    L = Hh * W
    ws = [rng.standard_normal((C, C)) * 0.5 for _ in range(4)]
    bo = rng.standard_normal(C)
    att = oracle.DisplacedSelfAttention(N, W, heads, *ws, bo)
    k_prev, v_prev = rng.standard_normal((L, C)), rng.standard_normal((L, C))
    att.prev = (k_prev, v_prev)
    t = rng.standard_normal((L, C))
    y = att(t, False)
    q, k, v = t @ ws[0].T, t @ ws[1].T, t @ ws[2].T
    P = L // N
    for p in range(N):
        own = slice(p * P, (p + 1) * P)
        others = np.r_[0:p * P, (p + 1) * P:L]
        K = np.concatenate([k[own], k_prev[others]])      # fresh own first, then stale others
        V = np.concatenate([v[own], v_prev[others]])
        o = np.zeros((P, C))
        for h in range(heads):
            c = slice(h * d, (h + 1) * d)
            o[:, c] = F.scaled_dot_product_attention(
                torch.from_numpy(q[own, c])[None], torch.from_numpy(K[:, c])[None],
                torch.from_numpy(V[:, c])[None])[0].numpy()
        _close(y[own], o @ ws[3].T + bo)


def test_sampled_query_tokens_match_full():
    cfg = SMALL
    wl = inputs.SyntheticWorkload(cfg)
    a, b = _block(cfg, wl), _block(cfg, wl)
    x0, x1 = wl.x(0), wl.x(1)
    a.step(x0, 0, 1)
    b.step(x0, 0, 1)
    tok = np.array([0, 5, 13, 17, 30, 47])
    full = a.step(x1, 1, 0)["y"]
    part = b.step(x1, 1, 0, query_tokens=tok)["y"]
    _close(part, full[tok])


def test_step_depends_only_on_previous_cache():
    cfg = SMALL
    wa = inputs.SyntheticWorkload(cfg, seed=0)
    wb = inputs.SyntheticWorkload(cfg, seed=0)
    a, b = _block(cfg, wa), _block(cfg, wb)
    a.step(wa.x(0), 0, 1)
    a.step(wa.x(1), 1, 0)
    b.step(wb.x(0) * 0.5 + 1.0, 0, 1)              # a different history
    b.step(wb.x(1) * -1.0, 1, 0)
    for name in ("gn1", "conv1", "gn2", "attn"):
        getattr(b, name).prev = copy.deepcopy(getattr(a, name).prev)
    x2 = wa.x(2)
    _close(b.step(x2, 2, 0)["y"], a.step(x2, 2, 0)["y"], tol=0)


def test_step_protocol_errors():
    cfg = SMALL
    wl = inputs.SyntheticWorkload(cfg)
    blk = _block(cfg, wl)
    with pytest.raises(RuntimeError):
        blk.step(wl.x(0), 0, 0)
    blk.step(wl.x(0), 0, 1)
    with pytest.raises(RuntimeError):
        blk.step(wl.x(1), 2, 0)


# --------------------------------------------------------------------------- brute force

def _brute_res_attn(xs, syncs, w, cfg):
    """Direct loops over every index: GN moments, GN merge, conv taps, Q/K/V, softmax."""
    H, W, C, N, G = cfg["H"], cfg["W"], cfg["C"], cfg["n_patches"], cfg["gn_groups"]
    heads, eps = cfg["heads"], cfg["gn_eps"]
    d, R, cg = C // heads, H // N, C // G
    prev = None
    outs = []

    def moments(x):
        m = np.zeros((N, G, 2))
        for p in range(N):
            for g in range(G):
                s1 = s2 = n = 0.0
                for i in range(p * R, (p + 1) * R):
                    for j in range(W):
                        for c in range(g * cg, (g + 1) * cg):
                            s1 += x[i, j, c]
                            s2 += x[i, j, c] ** 2
                            n += 1
                m[p, g] = (s1 / n, s2 / n)
        return m

    def gnorm(x, m, mprev, sync, gam, bet, act):
        out = np.zeros_like(x)
        for p in range(N):
            for g in range(G):
                if sync:
                    mu = sum(m[j, g, 0] for j in range(N)) / N
                    e2 = sum(m[j, g, 1] for j in range(N)) / N
                else:
                    mu = sum(mprev[j, g, 0] for j in range(N)) / N + m[p, g, 0] - mprev[p, g, 0]
                    e2 = sum(mprev[j, g, 1] for j in range(N)) / N + m[p, g, 1] - mprev[p, g, 1]
                var = max(e2 - mu * mu, 0.0)
                for i in range(p * R, (p + 1) * R):
                    for j in range(W):
                        for c in range(g * cg, (g + 1) * cg):
                            v = (x[i, j, c] - mu) / math.sqrt(var + eps) * gam[c] + bet[c]
                            out[i, j, c] = v / (1 + math.exp(-v)) if act else v
        return out

    for x, sync in zip(xs, syncs):
        x = x.astype(np.float64)
        m1 = moments(x)
        y1 = gnorm(x, m1, prev and prev["m1"], sync, w["gn1.weight"], w["gn1.bias"], True)
        h = np.zeros((H, W, C))
        wc, bc = w["conv1.weight"], w["conv1.bias"]
        for p in range(N):
            for i in range(p * R, (p + 1) * R):
                for j in range(W):
                    for co in range(C):
                        acc = bc[co]
                        for ci in range(C):
                            for r in range(3):
                                for s in range(3):
                                    ii, jj = i + r - 1, j + s - 1
                                    if not (0 <= ii < H and 0 <= jj < W):
                                        continue
                                    own = p * R <= ii < (p + 1) * R
                                    src = y1 if (own or sync) else prev["y1"]
                                    acc += wc[co, ci, r, s] * src[ii, jj, ci]
                        h[i, j, co] = acc
        m2 = moments(h)
        t = gnorm(h, m2, prev and prev["m2"], sync, w["gn2.weight"], w["gn2.bias"], False)
        L = H * W
        tok = t.reshape(L, C)
        q, k, v = (np.array([[sum(tok[l, c] * w[n][o, c] for c in range(C)) for o in range(C)]
                             for l in range(L)]) for n in ("attn.to_q.weight", "attn.to_k.weight",
                                                          "attn.to_v.weight"))
        o = np.zeros((L, C))
        for l in range(L):
            p = l // (R * W)
            for hd in range(heads):
                cs = range(hd * d, (hd + 1) * d)
                sc = []
                for m in range(L):
                    mine = m // (R * W) == p
                    kk = k if (mine or sync) else prev["k"]
                    sc.append(sum(q[l, c] * kk[m, c] for c in cs) / math.sqrt(d))
                mx = max(sc)
                e = [math.exp(s_ - mx) for s_ in sc]
                z = sum(e)
                for c in cs:
                    acc = 0.0
                    for m in range(L):
                        mine = m // (R * W) == p
                        vv = v if (mine or sync) else prev["v"]
                        acc += e[m] * vv[m, c]
                    o[l, c] = acc / z
        wo, bo = w["attn.to_out.weight"], w["attn.to_out.bias"]
        y = np.array([[bo[a] + sum(o[l, c] * wo[a, c] for c in range(C)) for a in range(C)]
                      for l in range(L)])
        outs.append(y)
        prev = dict(m1=m1, m2=m2, y1=y1, k=k, v=v)
    return outs


def test_brute_force_tiny_block():
    cfg = dict(name="tiny", H=4, W=3, C=4, n_patches=2, gn_groups=2, gn_eps=1e-5, heads=2,
               head_dim=2, dtype="f32", block="res_attn", steps=3, n_sync=1)
    wl = inputs.SyntheticWorkload(cfg, random_affine=True, weight_scale={
        "conv1.weight": 20.0, "attn.to_q.weight": 50.0, "attn.to_k.weight": 50.0,
        "attn.to_v.weight": 20.0})
    rng = np.random.default_rng(9)
    xs = [rng.standard_normal((4, 3, 4)) * (1 + t) for t in range(3)]
    syncs = [1, 0, 0]
    ref = _brute_res_attn(xs, syncs, {k: v.astype(np.float64) for k, v in wl.weights.items()}, cfg)
    blk = _block(cfg, wl)
    for t in range(3):
        _close(blk.step(xs[t], t, syncs[t])["y"], ref[t], tol=1e-11)


# --------------------------------------------------------------------------- transformer stage

def test_stage_sync_and_stale_equal_fresh():
    cfg = STAGE
    wl = inputs.SyntheticWorkload(cfg, random_affine=True)
    blk = _block(cfg, wl)
    x = wl.x(0)
    ref = _full(cfg, x.astype(np.float64), wl)["y"]
    _close(blk.step(x, 0, 1)["y"], ref)
    _close(blk.step(x, 1, 0)["y"], ref)


def test_stage_n1_displaced_equals_full():
    cfg = configs.get(STAGE, n_patches=1)
    wl = inputs.SyntheticWorkload(cfg)
    blk = _block(cfg, wl)
    for t in range(3):
        x = wl.x(t)
        _close(blk.step(x, t, int(t == 0))["y"], _full(cfg, x.astype(np.float64), wl)["y"])


# --------------------------------------------------------------------------- inputs

def test_inputs_deterministic_and_representable():
    cfg = configs.get(SMALL, dtype="bf16")
    a, b = inputs.SyntheticWorkload(cfg), inputs.SyntheticWorkload(cfg)
    for k in a.weights:
        assert np.array_equal(a.weights[k], b.weights[k])
        assert np.array_equal(inputs.round_to(a.weights[k], "bf16"), a.weights[k])
    for t in range(3):
        xa, xb = a.x(t), b.x(t)
        assert np.array_equal(xa, xb)
        assert np.array_equal(inputs.round_to(xa, "bf16"), xa)
    with pytest.raises(ValueError):
        a.x(7)
    assert a.schedule()[:2] == [(0, 1), (1, 0)]
