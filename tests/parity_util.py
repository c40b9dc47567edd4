"""Drive the CUDA path and the oracle side by side on the same seeded inputs."""
import numpy as np
import torch

import oracle
from patch_diffusion_unet_b200 import inputs

TOL = {"f32": 1e-5, "bf16": 2e-2}


def rel_l2(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_abs(a, b):
    return float(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)).max())


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def gpu_stage_views(blk, cfg):
    """Internal buffers of the last GPU step, reshaped like the oracle's intermediates
    (with a leading image axis for a batch; the slab keeps its [B*N, R+2, W, C] rows)."""
    H, W, C, N, heads = cfg["H"], cfg["W"], cfg["C"], cfg["n_patches"], cfg["heads"]
    B = cfg.get("batch", 1)
    R, L = H // N, H * W
    lead = (B,) if B > 1 else ()
    slab = host(blk.buffer("slab")).reshape(B * N, R + 2, W, C)
    out = dict(
        slab=slab,
        y1=slab[:, 1:R + 1].reshape(lead + (H, W, C)),
        h=host(blk.buffer("h")).reshape(lead + (H, W, C)),
        t=host(blk.buffer("t")).reshape(lead + (H, W, C)),
        o=host(blk.buffer("o")).reshape(lead + (L, C)),
        y=host(blk.buffer("y")).reshape(lead + (L, C)),
    )
    for n in ("q", "k", "v"):
        out[n] = host(blk.buffer(n)).reshape(heads, B, L, 64).transpose(1, 2, 0, 3).reshape(lead + (L, C))
    return out


def run_parity(cfg, n_steps, oracle_from=0, query_tokens=None, gn_mode=0, context=0, family=None,
               weight_scale=None, random_affine=False, stages=True, seed=0, x_fn=None, orc_out=None,
               kv_budget=None):
    """Run steps 0..n_steps-1 on the GPU; the oracle joins at step `oracle_from` (which must be
    a sync step, so no earlier state is needed) and is compared at every step from there.
    x_fn(t, x) -> x' changes the workload's input of step t before both sides see it (values
    exactly representable in the storage type).  orc_out, a list, receives the oracle's
    per-step outputs.  kv_budget sets the attention's K/V budget (1: whole-unit rounds wherever
    there are enough units).  Returns a list of per-step dicts {stage: (rel_l2, max_abs)}."""
    from patch_diffusion_unet_b200 import dfp

    wl = inputs.SyntheticWorkload(cfg, seed=seed, weight_scale=weight_scale, random_affine=random_affine)
    blk = dfp.DisplacedPatchBlock(cfg, gn_mode=gn_mode, context=context)
    if family is not None:
        blk.set_kernel_family(family)
    if kv_budget is not None:
        blk.set_attention_kv_budget(kv_budget)
    blk.load_weights(wl.weights)
    omode = ["corrected", "stale_others", "sync", "separate"][gn_mode]
    octx = ["displaced", "naive"][context]
    orc = oracle.make_block(cfg, wl.weights, wl.context, gn_mode=omode, context=octx)
    sched = wl.schedule()[:n_steps]
    assert sched[oracle_from][1] == 1, "the oracle must join on a synchronous step"
    results = []
    prev_slab = None
    for t, is_sync in sched:
        x = wl.x(t)
        if x_fn is not None:
            x = x_fn(t, x)
        xd = inputs.to_torch(x, cfg["dtype"]).cuda()
        blk.step(xd, t, is_sync)
        blk.check_device()
        if t < oracle_from:
            if stages:
                prev_slab = gpu_stage_views(blk, cfg)["slab"]
            continue
        ref = orc.step(x, t - oracle_from, is_sync, query_tokens=query_tokens)
        if orc_out is not None:
            orc_out.append(ref)
        g = gpu_stage_views(blk, cfg) if stages else dict(y=host(blk.output()))
        res = {}
        qsel = (query_tokens,) if cfg.get("batch", 1) == 1 else (slice(None), query_tokens)
        yg = g["y"] if query_tokens is None else g["y"][qsel]
        res["y"] = (rel_l2(yg, ref["y"]), max_abs(yg, ref["y"]))
        if stages:
            for n in ("y1", "h", "t", "q", "k", "v"):
                res[n] = (rel_l2(g[n], ref[n]), max_abs(g[n], ref[n]))
            og = g["o"] if query_tokens is None else g["o"][qsel]
            res["o"] = (rel_l2(og, ref["o"]), max_abs(og, ref["o"]))
            res["halo_ok"] = check_halos(cfg, g["slab"], prev_slab, is_sync, context)
            prev_slab = g["slab"]
        res["step"] = t
        res["sync"] = is_sync
        results.append(res)
    blk.close()
    return results


def check_halos(cfg, slab, prev_slab, is_sync, context):
    """Halo rows are copies: bit-exact against the source rows (stale = previous GPU step).
    A batch's slab holds B images of N patches each; every image is checked on its own
    (its first and last patch get zero halos: the image edges)."""
    N = cfg["n_patches"]
    B = cfg.get("batch", 1)
    if B > 1:
        per = slab.shape[0] // B
        return all(check_halos(dict(cfg, batch=1), slab[b * per:(b + 1) * per],
                               None if prev_slab is None else prev_slab[b * per:(b + 1) * per], is_sync, context)
                   for b in range(B))
    R = cfg["H"] // N
    if N == 1 or context == 1:
        return bool(np.all(slab[:, 0] == 0) and np.all(slab[:, R + 1] == 0))
    src = slab if is_sync else prev_slab
    if src is None:
        return True
    ok = np.all(slab[0, 0] == 0) and np.all(slab[N - 1, R + 1] == 0)
    for p in range(N):
        if p > 0:
            ok &= np.array_equal(slab[p, 0], src[p - 1, R])
        if p < N - 1:
            ok &= np.array_equal(slab[p, R + 1], src[p + 1, 1])
    return bool(ok)


def worst(results, key="y"):
    return max(r[key][0] for r in results)
