"""The five named workloads of the displaced-patch layer step.

Each workload is a plain dict of sizes; nothing here computes anything of the
method.  Shapes follow the pages' subject (SDXL latent levels, "DistriFusion:
Distributed Parallel Inference for High-Resolution Diffusion Models" project
README, Performance section: 1024/2048/3840 px images).

Keys
----
name        short workload name used in reports
H, W, C     latent feature map (rows, columns, channels), NHWC, batch 1
n_patches   number of row patches N (patch p owns rows [p*H/N, (p+1)*H/N))
gn_groups   GroupNorm groups G;  gn_eps the GroupNorm epsilon
heads, head_dim   self-attention heads x head width (heads*head_dim == C)
dtype       storage / MMA operand type ("f32" or "bf16")
block       "res_attn" (GN+SiLU, conv3x3, GN, self-attention),
            "sdxl_stage" (ResNet block + transformer blocks)
            or "unet" (the multi-level UNet of a whole denoising step)
steps, n_sync     denoising steps in a run and how many of the first are synchronous
n_xformer, ffn_inner, ctx_len, ctx_dim   transformer-stage extras (sdxl_stage only)
widths, latent_c    UNet level widths (full, half, quarter resolution) and latent channels;
ddim_train_steps, beta_start, beta_end   the DDIM schedule (unet only)
"""

CONFIGS = {
    0: dict(name="tiny-16x16x64-n2-fp32", H=16, W=16, C=64, n_patches=2, gn_groups=8,
            gn_eps=1e-5, heads=1, head_dim=64, dtype="f32", block="res_attn",
            steps=4, n_sync=1),
    1: dict(name="sdxl1024-64x64x640-n4-bf16", H=64, W=64, C=640, n_patches=4, gn_groups=32,
            gn_eps=1e-5, heads=10, head_dim=64, dtype="bf16", block="res_attn",
            steps=50, n_sync=5),
    2: dict(name="sdxl2048-128x128x640-n8-bf16", H=128, W=128, C=640, n_patches=8, gn_groups=32,
            gn_eps=1e-5, heads=10, head_dim=64, dtype="bf16", block="res_attn",
            steps=50, n_sync=5),
    3: dict(name="sdxl3840-240x240x640-n8-bf16", H=240, W=240, C=640, n_patches=8, gn_groups=32,
            gn_eps=1e-5, heads=10, head_dim=64, dtype="bf16", block="res_attn",
            steps=10, n_sync=2),
    4: dict(name="sdxl-stage-64x64x1280-n8-bf16", H=64, W=64, C=1280, n_patches=8, gn_groups=32,
            gn_eps=1e-5, heads=20, head_dim=64, dtype="bf16", block="sdxl_stage",
            steps=50, n_sync=5, n_xformer=2, ffn_inner=5120, ctx_len=77, ctx_dim=2048),
    # the multi-level UNet of a 1024 px image and its 50-step DDIM loop (latent 128x128x4;
    # levels 128^2 / 64^2 / 32^2 with 320 / 640 / 1280 channels, 8 row patches at every level)
    5: dict(name="sdxl-unet-1024-128x128-n8-bf16", H=128, W=128, C=320, n_patches=8, gn_groups=32,
            gn_eps=1e-5, heads=5, head_dim=64, dtype="bf16", block="unet", steps=50, n_sync=5,
            widths=(320, 640, 1280), latent_c=4, ctx_len=77, ctx_dim=2048,
            ddim_train_steps=1000, beta_start=0.00085, beta_end=0.012),
}


def get(cfg_id_or_dict, **overrides):
    """Return a copy of a named workload (by id) or of a dict, with overrides applied."""
    base = CONFIGS[cfg_id_or_dict] if isinstance(cfg_id_or_dict, int) else cfg_id_or_dict
    out = dict(base)
    out.update(overrides)
    return out


def tokens(cfg):
    return cfg["H"] * cfg["W"]


def rows_per_patch(cfg):
    return cfg["H"] // cfg["n_patches"]
