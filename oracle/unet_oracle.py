"""Oracle of a displaced-patch multi-level UNet and its DDIM loop (numpy fp64, CPU).

TEST INFRASTRUCTURE ONLY, like dfp_oracle: only the tests, ``__graft_entry__.smoke()``
and the benchmark's CPU legs may import or run it; it shares no code with the CUDA path.

The pages run SDXL's UNet for 50 DDIM steps with every convolution, GroupNorm and
self-attention of the UNet replaced by its displaced-patch form, the latent split into
the same row patches at every resolution ("DistriFusion: Distributed Parallel Inference
for High-Resolution Diffusion Models" README, Overview (c) and Performance; paper
reading blog, Implementation details: 50-step DDIM, warm-up steps synchronous; source
walkthrough, Patch Parallelism: DistriUNetPP wraps every conv, norm and attention layer).
No weights are available, so the network is random and SDXL-shaped.  Readings adopted:

  R9   UNet shape (the pages name SDXL, print no architecture): latent [H, W, 4];
       levels at H, H/2, H/4 with widths c0, c1, c2 (SDXL at 1024 px: 128^2, 64^2, 32^2 with
       320, 640, 1280 channels); one ResNet block per level, a transformer block (the
       layer stage's: pre-LayerNorm self-attention on displaced K/V, cross-attention to a
       fixed context, GEGLU feed-forward, all residual) at the two lower levels; a
       stride-2 3x3 conv between levels down, nearest x2 upsampling and a 3x3 conv up,
       the down path's level outputs concatenated (channels: upsampled, then skip) into
       the up path's ResNet blocks.  ResNet(x): h = conv1(SiLU(GN1(x))) + the timestep
       embedding projected to the block's width; h = conv2(SiLU(GN2(h))); h + x, or h +
       a 1x1 projection of x when the width changes.  Timestep embedding: [cos(tau f_k),
       sin(tau f_k)], f_k = 10000^(-k/(c0/2)), k < c0/2, then Linear(c0 -> 4 c0), SiLU,
       Linear(4 c0 -> 4 c0); each ResNet adds Linear(4 c0 -> width)(SiLU(embedding)).
       Output: conv_out(SiLU(GN(h))) -> 4 channels, the predicted noise.
  R10  DDIM (eta = 0) on a scaled-linear beta schedule of 1000 training steps
       (beta_i = (sqrt(b0) + i (sqrt(b1) - sqrt(b0)) / 999)^2, alpha_bar_i = prod_{j<=i}
       (1 - beta_j)), 50 evenly spaced timesteps tau_k = k * 1000 / 50 + 1 visited from
       the largest down: x_prev = sqrt(ab_prev) x0_hat + sqrt(1 - ab_prev) eps,
       x0_hat = (x - sqrt(1 - ab) eps) / sqrt(ab), ab_prev = 1 after the last step.
  R11  Displacement at every resolution: patch p owns rows [p H_l / N, (p+1) H_l / N) at
       each level; each displaced layer keeps its own previous-step state (R1-R4 of
       dfp_oracle).  The stride-2 conv of patch p reads its own input rows and the one row
       above (from the previous step on displaced steps); the upsampling is per patch
       (local), and its conv reads halo rows of the upsampled map like any conv.
"""
import numpy as np

from .dfp_oracle import (CTX_DISPLACED, GN_CORRECTED, CrossAttention, DisplacedConv3x3,
                         DisplacedGroupNorm, DisplacedSelfAttention, _StepProtocol, gelu_erf,
                         layer_norm, patch_bounds)


def silu(y):
    return y / (1.0 + np.exp(-y))


# ----------------------------------------------------------------------------- schedule

def alphas_cumprod(n_train=1000, beta_start=0.00085, beta_end=0.012):
    """alpha_bar of the scaled-linear schedule (R10)."""
    betas = np.linspace(np.sqrt(beta_start), np.sqrt(beta_end), n_train) ** 2
    return np.cumprod(1.0 - betas)


def ddim_timesteps(n_steps=50, n_train=1000):
    """The visited timesteps, largest first (R10)."""
    ratio = n_train // n_steps
    return (np.arange(n_steps) * ratio + 1)[::-1]


def ddim_step(x, eps, ab, ab_prev):
    """One deterministic DDIM update (R10)."""
    x0 = (x - np.sqrt(1.0 - ab) * eps) / np.sqrt(ab)
    return np.sqrt(ab_prev) * x0 + np.sqrt(1.0 - ab_prev) * eps


def timestep_embedding(tau, dim):
    """[cos(tau f_k), sin(tau f_k)], f_k = 10000^(-k / (dim/2)) (R9)."""
    half = dim // 2
    f = np.exp(-np.log(10000.0) * np.arange(half) / half)
    return np.concatenate([np.cos(tau * f), np.sin(tau * f)])


# ----------------------------------------------------------------------------- layers

class DisplacedDownsample:
    """3x3 conv with stride 2 over N row patches (R11): output rows of patch p are computed
    from its own input rows and the row above, which comes from the previous step's input
    map on displaced steps; zero padding at the image edges and left/right."""

    def __init__(self, N, weight, bias):
        self.N = N
        self.weight, self.bias = np.asarray(weight, np.float64), np.asarray(bias, np.float64)
        self.prev = None

    def __call__(self, y, is_sync):
        H, W, _ = y.shape
        if not is_sync and self.prev is None:
            raise RuntimeError("displaced downsample needs the previous step's input map")
        src = y if is_sync else self.prev
        Co = self.weight.shape[0]
        out = np.empty((H // 2, W // 2, Co))
        for r0, r1 in patch_bounds(H, self.N):
            top = src[r0 - 1:r0] if r0 > 0 else np.zeros((1,) + y.shape[1:])
            band = np.concatenate([top, y[r0:r1]])                      # rows r0-1 .. r1-1
            band = np.pad(band, ((0, 0), (1, 1), (0, 0)))               # zero columns left/right
            o = np.zeros(((r1 - r0) // 2, W // 2, Co)) + self.bias
            for r in range(3):
                for s in range(3):
                    # output row i (patch-local) reads band row 2i + r, column 2j + s
                    o += band[r:r + (r1 - r0):2, s:s + W:2, :] @ self.weight[:, :, r, s].T
            out[r0 // 2:r1 // 2] = o
        self.prev = y
        return out


def upsample_nearest(y):
    return np.repeat(np.repeat(y, 2, axis=0), 2, axis=1)


class ResNet:
    def __init__(self, N, G, eps, w, p, gn_mode, context):
        self.gn1 = DisplacedGroupNorm(N, G, eps, w[p + "norm1.weight"], w[p + "norm1.bias"], gn_mode, context, silu=True)
        self.conv1 = DisplacedConv3x3(N, w[p + "conv1.weight"], w[p + "conv1.bias"], context)
        self.gn2 = DisplacedGroupNorm(N, G, eps, w[p + "norm2.weight"], w[p + "norm2.bias"], gn_mode, context, silu=True)
        self.conv2 = DisplacedConv3x3(N, w[p + "conv2.weight"], w[p + "conv2.bias"], context)
        self.wt, self.bt = w[p + "time_emb_proj.weight"], w[p + "time_emb_proj.bias"]
        self.sc = (w[p + "conv_shortcut.weight"], w[p + "conv_shortcut.bias"]) if p + "conv_shortcut.weight" in w \
            else None

    def __call__(self, x, temb_act, is_sync):
        h = self.conv1(self.gn1(x, is_sync), is_sync) + (self.wt @ temb_act + self.bt)
        h = self.conv2(self.gn2(h, is_sync), is_sync)
        if self.sc is None:
            return x + h
        return x @ self.sc[0].T + self.sc[1] + h


class TransformerBlock:
    """The layer stage's transformer block on a map [H, W, C] (R9)."""

    def __init__(self, N, W, heads, w, p, ctx, context):
        self.w, self.p = w, p
        self.sa = DisplacedSelfAttention(N, W, heads, w[p + "attn1.to_q.weight"], w[p + "attn1.to_k.weight"],
                                         w[p + "attn1.to_v.weight"], w[p + "attn1.to_out.weight"],
                                         w[p + "attn1.to_out.bias"], context)
        self.ca = CrossAttention(heads, w[p + "attn2.to_q.weight"], w[p + "attn2.to_k.weight"],
                                 w[p + "attn2.to_v.weight"], w[p + "attn2.to_out.weight"], w[p + "attn2.to_out.bias"],
                                 ctx)

    def __call__(self, x, is_sync):
        w, p = self.w, self.p
        H, W, C = x.shape
        r = x.reshape(H * W, C)
        r = r + self.sa(layer_norm(r, w[p + "norm1.weight"], w[p + "norm1.bias"]), is_sync)
        r = r + self.ca(layer_norm(r, w[p + "norm2.weight"], w[p + "norm2.bias"]))
        u = layer_norm(r, w[p + "norm3.weight"], w[p + "norm3.bias"])
        hg = u @ w[p + "ff.proj.weight"].T + w[p + "ff.proj.bias"]
        F = hg.shape[1] // 2
        r = r + (hg[:, :F] * gelu_erf(hg[:, F:])) @ w[p + "ff.out.weight"].T + w[p + "ff.out.bias"]
        return r.reshape(H, W, C)


# ----------------------------------------------------------------------------- the UNet

class DisplacedUNet(_StepProtocol):
    """The SDXL-shaped UNet of R9 with every conv, GroupNorm and self-attention displaced
    (R11); step() returns the predicted noise for latent x [H, W, latent_c] at timestep tau."""

    def __init__(self, cfg, weights, context_tokens, gn_mode=GN_CORRECTED, context=CTX_DISPLACED):
        N, G, eps = cfg["n_patches"], cfg["gn_groups"], cfg["gn_eps"]
        c0, c1, c2 = cfg["widths"]
        W = cfg["W"]
        w = {k: np.asarray(v, np.float64) for k, v in weights.items()}
        self.cfg, self.w, self.c0 = cfg, w, c0
        ctx = np.asarray(context_tokens, np.float64)
        self.conv_in = DisplacedConv3x3(N, w["conv_in.weight"], w["conv_in.bias"], context)
        args = (N, G, eps, w)
        self.res0 = ResNet(*args, "down0.resnet.", gn_mode, context)
        self.down0 = DisplacedDownsample(N, w["down0.downsample.weight"], w["down0.downsample.bias"])
        self.res1 = ResNet(*args, "down1.resnet.", gn_mode, context)
        self.xf1 = TransformerBlock(N, W // 2, c1 // 64, w, "down1.xf.", ctx, context)
        self.down1 = DisplacedDownsample(N, w["down1.downsample.weight"], w["down1.downsample.bias"])
        self.res2 = ResNet(*args, "down2.resnet.", gn_mode, context)
        self.xf2 = TransformerBlock(N, W // 4, c2 // 64, w, "down2.xf.", ctx, context)
        self.up1 = DisplacedConv3x3(N, w["up1.upsample.weight"], w["up1.upsample.bias"], context)
        self.ures1 = ResNet(*args, "up1.resnet.", gn_mode, context)
        self.uxf1 = TransformerBlock(N, W // 2, c1 // 64, w, "up1.xf.", ctx, context)
        self.up0 = DisplacedConv3x3(N, w["up0.upsample.weight"], w["up0.upsample.bias"], context)
        self.ures0 = ResNet(*args, "up0.resnet.", gn_mode, context)
        self.gn_out = DisplacedGroupNorm(N, G, eps, w["norm_out.weight"], w["norm_out.bias"], gn_mode, context,
                                         silu=True)
        self.conv_out = DisplacedConv3x3(N, w["conv_out.weight"], w["conv_out.bias"], context)
        self.last_step = None

    def temb(self, tau):
        w = self.w
        e = timestep_embedding(float(tau), self.c0)
        h = silu(w["time_embedding.linear_1.weight"] @ e + w["time_embedding.linear_1.bias"])
        return w["time_embedding.linear_2.weight"] @ h + w["time_embedding.linear_2.bias"]

    def step(self, x, step, is_sync, tau):
        self._check(step, is_sync)
        x = np.asarray(x, np.float64)
        ta = silu(self.temb(tau))
        out = {}
        h = self.conv_in(x, is_sync)
        s0 = h = self.res0(h, ta, is_sync)
        h = self.down0(h, is_sync)
        h = self.res1(h, ta, is_sync)
        s1 = h = self.xf1(h, is_sync)
        h = self.down1(h, is_sync)
        h = self.res2(h, ta, is_sync)
        h = self.xf2(h, is_sync)
        out["mid"] = h
        h = self.up1(upsample_nearest(h), is_sync)
        h = self.ures1(np.concatenate([h, s1], axis=-1), ta, is_sync)
        h = self.uxf1(h, is_sync)
        h = self.up0(upsample_nearest(h), is_sync)
        h = self.ures0(np.concatenate([h, s0], axis=-1), ta, is_sync)
        out["eps"] = self.conv_out(self.gn_out(h, is_sync), is_sync)
        out.update(s0=s0, s1=s1, up0=h)
        return out


def ddim_sample(unet, x_T, n_steps, n_sync, n_train=1000, beta_start=0.00085, beta_end=0.012, stop=None):
    """DDIM (R10) from x_T with the displaced UNet: the first n_sync steps synchronous.
    Returns the list of latents x after each step (stop: run only that many steps)."""
    acp = alphas_cumprod(n_train, beta_start, beta_end)
    taus = ddim_timesteps(n_steps, n_train)
    x = np.asarray(x_T, np.float64)
    xs = []
    for k, tau in enumerate(taus[:stop]):
        eps = unet.step(x, k, int(k < n_sync), tau)["eps"]
        ab_prev = acp[taus[k + 1]] if k + 1 < len(taus) else 1.0
        x = ddim_step(x, eps, acp[tau], ab_prev)
        xs.append(x)
    return xs
