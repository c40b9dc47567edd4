"""Oracle: a plain, slow, fp64 CPU restatement of the displaced-patch UNet layer step.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import or run this module.  It
shares no code with the CUDA path (no kernels, helpers, tables or constants),
and the product path never calls it.

What it computes, and where the pages say so
--------------------------------------------
Sources are web pages about DistriFusion (CVPR 2024):
  [README]  "DistriFusion: Distributed Parallel Inference for High-Resolution
            Diffusion Models" project README (dongaigc.com mirror)
  [WALK]    "DistriFusion源码探秘：从DistriUNetPP到DistriAttentionTP的模块设计原理"
            source walkthrough (jsqmd.com)
  [CSDN]    "阅读论文1" paper-reading blog post (blog.csdn.net)
  [MEENS]   meens.ai catalogue page on DistriFusion

* The latent is split into N patches, one per device; each device computes
  its own patch ([README] Overview (c); [WALK] "Patch Parallelism的实现原理";
  [MEENS] section 2).  Patches here are contiguous row bands.
* The first step(s) use synchronous patch interaction; afterwards each patch
  reuses the previous step's activations of the other patches as context
  ([README] Overview (c); [CSDN] Implementation details: step 0 plus 4 more
  warm-up steps are synchronous; [MEENS] section 2).
* Three kinds of layers are wrapped ([WALK] items 1-3): the convolution
  (DistriConv2dPP), self-/cross-attention (DistriSelfAttentionPP /
  DistriCrossAttentionPP) and GroupNorm (DistriGroupNorm).  Linear layers and
  LayerNorm act per token and need no context.
* GroupNorm defaults to a "corrected asynchronous" mode ([README] Benchmarks,
  ``--sync_mode`` flag).  The pages name the mode but print no formula.

Readings adopted where the pages are silent:
  R1  conv3x3 context: the one row above / below a patch comes from the
      previous step's conv-input map on displaced steps, from the current map
      on synchronous steps; zero outside the image; zero padding left/right.
  R2  attention context: a patch's queries attend to its own fresh K/V and to
      every other patch's K/V from the previous step (current on sync steps).
  R3  GroupNorm "corrected": with per-(patch, group) moments m = (E[x], E[x^2]),
      est_p = mean_j m_j^{t-1} + (m_p^t - m_p^{t-1}); var = max(E2 - mu^2, 0).
      Alternative "stale_others": est_p = (m_p^t + sum_{j!=p} m_j^{t-1}) / N.
      Sync steps use the exact full-map moments.  Variance is biased (/n).
  R4  every step (sync ones included) refreshes the context caches with the
      values it computed; a displaced step reads only the caches of step t-1.
  R5  Q/K/V projections carry no bias; to_out carries one; the res-attn block
      output is the attention output without a residual add.
  R6  "naive" context (the pages' naive-patch baseline, [README] Overview (b);
      [CSDN] Baselines): no cross-patch context at all -- zero halo rows,
      patch-local GroupNorm moments, attention within the patch only.
  R7  guidance batch (classifier-free guidance at scale 5, [CSDN] Implementation
      details; [README] Benchmarks, --no_split_batch): each image of a batch is
      its own displaced-patch step -- own GroupNorm statistics, halo rows, K/V
      and text context -- sharing only the weights and the step schedule.
  R8  GroupNorm-only variants of --sync_mode ([README] Benchmarks: the flag picks
      among GroupNorm synchronisation modes and names only the default): "sync" uses this step's
      moments of every patch (the exact full-map GroupNorm) on displaced steps too,
      "separate" uses only the patch's own moments of this step (patch-local
      GroupNorm) on displaced steps; conv halos and attention K/V stay displaced in
      both.  Sync steps are exact in every mode.
"""
import numpy as np

GN_CORRECTED = "corrected"
GN_STALE_OTHERS = "stale_others"
GN_SYNC = "sync"
GN_SEPARATE = "separate"
CTX_DISPLACED = "displaced"
CTX_NAIVE = "naive"


# ----------------------------------------------------------------------------
# elementary pieces

def patch_bounds(H, N):
    """Row range [r0, r1) of each of the N row patches ([WALK] patch split)."""
    if H % N:
        raise ValueError("H must be a multiple of the patch count")
    R = H // N
    return [(p * R, (p + 1) * R) for p in range(N)]


def group_moments(xp, G):
    """(E[x], E[x^2]) per channel group over every pixel of a patch xp [rows, W, C] -> [G, 2]."""
    rows, W, C = xp.shape
    g = xp.reshape(rows * W, G, C // G)
    return np.stack([g.mean(axis=(0, 2)), (g * g).mean(axis=(0, 2))], axis=-1)


def merge_moments(fresh, stale, is_sync, mode, context=CTX_DISPLACED):
    """Per-patch GroupNorm mean and variance from fresh / stale moments [N, G, 2] (R3, R6, R8)."""
    N = fresh.shape[0]
    if context == CTX_NAIVE or (mode == GN_SEPARATE and not is_sync):
        est = fresh
    elif is_sync or mode == GN_SYNC:
        est = np.broadcast_to(fresh.mean(axis=0), fresh.shape)
    elif mode == GN_CORRECTED:
        est = stale.mean(axis=0)[None] + (fresh - stale)
    elif mode == GN_STALE_OTHERS:
        est = (fresh + (stale.sum(axis=0)[None] - stale)) / N
    else:
        raise ValueError(mode)
    mu = est[..., 0]
    var = np.maximum(est[..., 1] - mu * mu, 0.0)
    return mu, var


def normalize(xp, mu_g, var_g, gamma, beta, eps):
    """(x - mu) / sqrt(var + eps) * gamma + beta with per-group mu, var broadcast to channels."""
    cg = xp.shape[-1] // mu_g.shape[0]
    mu_c = np.repeat(mu_g, cg)
    rstd_c = 1.0 / np.sqrt(np.repeat(var_g, cg) + eps)
    return (xp - mu_c) * rstd_c * gamma + beta


def silu(y):
    return y / (1.0 + np.exp(-y))


def gelu_erf(y):
    """Exact GELU, 0.5 y (1 + erf(y / sqrt 2)) (scipy's erf as the library step)."""
    from scipy.special import erf
    return 0.5 * y * (1.0 + erf(y / np.sqrt(2.0)))


def conv3x3_rows(inp, weight, bias):
    """3x3 convolution, stride 1, of a row band that already carries one context row
    above and below: inp [R+2, W, Ci] -> [R, W, Co]; zero padding left/right.
    weight [Co, Ci, 3, 3] (PyTorch layout), bias [Co]."""
    R = inp.shape[0] - 2
    W = inp.shape[1]
    padded = np.pad(inp, ((0, 0), (1, 1), (0, 0)))
    out = np.zeros((R, W, weight.shape[0])) + bias
    for r in range(3):
        for s in range(3):
            out += padded[r:r + R, s:s + W, :] @ weight[:, :, r, s].T
    return out


def softmax_attention(q, k, v, scale, chunk=256):
    """softmax(q k^T * scale) v with the row maximum subtracted; q [Lq, d], k, v [Lk, d]."""
    out = np.empty((q.shape[0], v.shape[1]))
    for i0 in range(0, q.shape[0], chunk):
        s = (q[i0:i0 + chunk] @ k.T) * scale
        s -= s.max(axis=1, keepdims=True)
        e = np.exp(s)
        out[i0:i0 + chunk] = (e @ v) / e.sum(axis=1, keepdims=True)
    return out


def layer_norm(x, gamma, beta, eps=1e-5):
    """Per-token LayerNorm over the channel axis (biased variance)."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * gamma + beta


# ----------------------------------------------------------------------------
# displaced layers, each holding its own previous-step context (R4)

class DisplacedGroupNorm:
    """GroupNorm over N row patches with stale cross-patch statistics (R3)
    ([WALK] item 3, DistriGroupNorm; [README] ``--sync_mode``)."""

    def __init__(self, N, G, eps, gamma, beta, mode=GN_CORRECTED, context=CTX_DISPLACED, silu=False):
        self.N, self.G, self.eps = N, G, eps
        self.gamma, self.beta = np.asarray(gamma, np.float64), np.asarray(beta, np.float64)
        self.mode, self.context, self.silu = mode, context, silu
        self.prev = None          # [N, G, 2] fresh moments of step t-1
        self.last = None          # (mu, var) used in the last call, [N, G] each

    def __call__(self, x, is_sync):
        H = x.shape[0]
        bounds = patch_bounds(H, self.N)
        fresh = np.stack([group_moments(x[r0:r1], self.G) for r0, r1 in bounds])
        reads_stale = self.mode in (GN_CORRECTED, GN_STALE_OTHERS) and self.context != CTX_NAIVE
        if not is_sync and reads_stale and self.prev is None:
            raise RuntimeError("displaced GroupNorm needs the previous step's statistics")
        mu, var = merge_moments(fresh, self.prev, is_sync, self.mode, self.context)
        out = np.empty_like(x)
        for p, (r0, r1) in enumerate(bounds):
            y = normalize(x[r0:r1], mu[p], var[p], self.gamma, self.beta, self.eps)
            out[r0:r1] = silu(y) if self.silu else y
        self.prev = fresh
        self.last = (mu, var)
        return out


class DisplacedConv3x3:
    """3x3 conv over N row patches whose one-row halos come from the previous
    step's input map on displaced steps (R1) ([WALK] item 1, DistriConv2dPP)."""

    def __init__(self, N, weight, bias, context=CTX_DISPLACED):
        self.N = N
        self.weight, self.bias = np.asarray(weight, np.float64), np.asarray(bias, np.float64)
        self.context = context
        self.prev = None          # full conv-input map of step t-1

    def __call__(self, y, is_sync):
        H, W, _ = y.shape
        if not is_sync and self.context != CTX_NAIVE and self.prev is None:
            raise RuntimeError("displaced conv needs the previous step's input map")
        src = y if is_sync else self.prev
        zero = np.zeros((1,) + y.shape[1:])
        out = np.empty((H, W, self.weight.shape[0]))
        for r0, r1 in patch_bounds(H, self.N):
            if self.context == CTX_NAIVE:
                top, bot = zero, zero
            else:
                top = src[r0 - 1:r0] if r0 > 0 else zero
                bot = src[r1:r1 + 1] if r1 < H else zero
            out[r0:r1] = conv3x3_rows(np.concatenate([top, y[r0:r1], bot]), self.weight, self.bias)
        self.prev = y
        return out


class DisplacedSelfAttention:
    """Multi-head self-attention over the tokens of N row patches; a patch's
    queries see its own fresh K/V and the other patches' K/V of step t-1 (R2)
    ([WALK] item 2, DistriSelfAttentionPP).  Tokens are row-major (h, w)."""

    def __init__(self, N, W, heads, wq, wk, wv, wo, bo, context=CTX_DISPLACED):
        self.N, self.W, self.heads = N, W, heads
        self.wq, self.wk, self.wv = (np.asarray(a, np.float64) for a in (wq, wk, wv))
        self.wo, self.bo = np.asarray(wo, np.float64), np.asarray(bo, np.float64)
        self.context = context
        self.prev = None          # (K, V) [L, C] of step t-1
        self.last = None

    def __call__(self, t, is_sync, query_tokens=None):
        """t [L, C] -> y [L, C] (or [len(query_tokens), C] for a token sample)."""
        L, C = t.shape
        d = C // self.heads
        if not is_sync and self.context != CTX_NAIVE and self.prev is None:
            raise RuntimeError("displaced attention needs the previous step's K/V")
        q, k, v = t @ self.wq.T, t @ self.wk.T, t @ self.wv.T
        H = L // self.W
        if query_tokens is None:
            query_tokens = np.arange(L)
        query_tokens = np.asarray(query_tokens)
        o = np.zeros((len(query_tokens), C))
        for r0, r1 in patch_bounds(H, self.N):
            a, b = r0 * self.W, r1 * self.W
            sel = np.nonzero((query_tokens >= a) & (query_tokens < b))[0]
            if len(sel) == 0:
                continue
            if self.context == CTX_NAIVE:
                kc, vc = k[a:b], v[a:b]
            elif is_sync:
                kc, vc = k, v
            else:
                kc, vc = self.prev[0].copy(), self.prev[1].copy()
                kc[a:b], vc[a:b] = k[a:b], v[a:b]
            qs = q[query_tokens[sel]]
            for h in range(self.heads):
                c = slice(h * d, (h + 1) * d)
                o[sel, c] = softmax_attention(qs[:, c], kc[:, c], vc[:, c], 1.0 / np.sqrt(d))
        self.prev = (k, v)
        self.last = dict(q=q, k=k, v=v, o=o)
        return o @ self.wo.T + self.bo


class CrossAttention:
    """Multi-head attention of the tokens to a fixed text context ([WALK] item 2,
    DistriCrossAttentionPP: the context is the same for every patch, so no staleness)."""

    def __init__(self, heads, wq, wk, wv, wo, bo, context):
        self.heads = heads
        ctx = np.asarray(context, np.float64)
        self.wq, self.wo, self.bo = (np.asarray(a, np.float64) for a in (wq, wo, bo))
        self.k = ctx @ np.asarray(wk, np.float64).T
        self.v = ctx @ np.asarray(wv, np.float64).T

    def __call__(self, t):
        L, C = t.shape
        d = C // self.heads
        q = t @ self.wq.T
        o = np.empty((L, C))
        for h in range(self.heads):
            c = slice(h * d, (h + 1) * d)
            o[:, c] = softmax_attention(q[:, c], self.k[:, c], self.v[:, c], 1.0 / np.sqrt(d))
        return o @ self.wo.T + self.bo


# ----------------------------------------------------------------------------
# blocks

class _StepProtocol:
    def _check(self, step, is_sync):
        if step == 0:
            if not is_sync:
                raise RuntimeError("step 0 must be synchronous")
        elif self.last_step is None or step != self.last_step + 1:
            raise RuntimeError(f"step {step} does not follow step {self.last_step}")
        self.last_step = step


class ResAttnBlock(_StepProtocol):
    """GN(+SiLU) -> conv3x3 -> GN -> self-attention, every layer displaced.

    weights: dict of float arrays named as in PyTorch modules (gn1.weight,
    conv1.weight [C, C, 3, 3], attn.to_q.weight [C, C], ...)."""

    def __init__(self, cfg, weights, gn_mode=GN_CORRECTED, context=CTX_DISPLACED):
        N, G, eps = cfg["n_patches"], cfg["gn_groups"], cfg["gn_eps"]
        w = {k: np.asarray(v, np.float64) for k, v in weights.items()}
        self.cfg = cfg
        self.gn1 = DisplacedGroupNorm(N, G, eps, w["gn1.weight"], w["gn1.bias"], gn_mode, context, silu=True)
        self.conv1 = DisplacedConv3x3(N, w["conv1.weight"], w["conv1.bias"], context)
        self.gn2 = DisplacedGroupNorm(N, G, eps, w["gn2.weight"], w["gn2.bias"], gn_mode, context, silu=False)
        self.attn = DisplacedSelfAttention(N, cfg["W"], cfg["heads"], w["attn.to_q.weight"],
                                           w["attn.to_k.weight"], w["attn.to_v.weight"],
                                           w["attn.to_out.weight"], w["attn.to_out.bias"], context)
        self.last_step = None

    def step(self, x, step, is_sync, query_tokens=None):
        """One layer step on x [H, W, C]; returns a dict of the output and every intermediate."""
        self._check(step, is_sync)
        x = np.asarray(x, np.float64)
        H, W, C = x.shape
        y1 = self.gn1(x, is_sync)
        h = self.conv1(y1, is_sync)
        t = self.gn2(h, is_sync)
        y = self.attn(t.reshape(H * W, C), is_sync, query_tokens)
        return dict(y=y, y1=y1, h=h, t=t, gn1=self.gn1.last, gn2=self.gn2.last, **self.attn.last)


class SDXLStage(_StepProtocol):
    """ResNet block (2x [GN + SiLU + conv3x3] plus residual) followed by
    transformer blocks (pre-LayerNorm self-attention on displaced K/V,
    cross-attention to a fixed context, GEGLU feed-forward), all residual."""

    def __init__(self, cfg, weights, context_tokens, gn_mode=GN_CORRECTED, context=CTX_DISPLACED):
        N, G, eps, C = cfg["n_patches"], cfg["gn_groups"], cfg["gn_eps"], cfg["C"]
        w = {k: np.asarray(v, np.float64) for k, v in weights.items()}
        self.cfg, self.w = cfg, w
        self.norm1 = DisplacedGroupNorm(N, G, eps, w["resnet.norm1.weight"], w["resnet.norm1.bias"],
                                        gn_mode, context, silu=True)
        self.conv1 = DisplacedConv3x3(N, w["resnet.conv1.weight"], w["resnet.conv1.bias"], context)
        self.norm2 = DisplacedGroupNorm(N, G, eps, w["resnet.norm2.weight"], w["resnet.norm2.bias"],
                                        gn_mode, context, silu=True)
        self.conv2 = DisplacedConv3x3(N, w["resnet.conv2.weight"], w["resnet.conv2.bias"], context)
        self.blocks = []
        for b in range(cfg["n_xformer"]):
            p = f"xf{b}."
            sa = DisplacedSelfAttention(N, cfg["W"], cfg["heads"], w[p + "attn1.to_q.weight"],
                                        w[p + "attn1.to_k.weight"], w[p + "attn1.to_v.weight"],
                                        w[p + "attn1.to_out.weight"], w[p + "attn1.to_out.bias"], context)
            ca = CrossAttention(cfg["heads"], w[p + "attn2.to_q.weight"], w[p + "attn2.to_k.weight"],
                                w[p + "attn2.to_v.weight"], w[p + "attn2.to_out.weight"],
                                w[p + "attn2.to_out.bias"], context_tokens)
            self.blocks.append((p, sa, ca))
        self.last_step = None

    def _ffn(self, p, u):
        w = self.w
        hg = u @ w[p + "ff.proj.weight"].T + w[p + "ff.proj.bias"]
        F = hg.shape[1] // 2
        return (hg[:, :F] * gelu_erf(hg[:, F:])) @ w[p + "ff.out.weight"].T + w[p + "ff.out.bias"]

    def step(self, x, step, is_sync):
        self._check(step, is_sync)
        x = np.asarray(x, np.float64)
        H, W, C = x.shape
        w = self.w
        h1 = self.conv1(self.norm1(x, is_sync), is_sync)
        h2 = self.conv2(self.norm2(h1, is_sync), is_sync)
        r = (x + h2).reshape(H * W, C)
        out = dict(resnet=r.reshape(H, W, C).copy())
        for p, sa, ca in self.blocks:
            r = r + sa(layer_norm(r, w[p + "norm1.weight"], w[p + "norm1.bias"]), is_sync)
            out[p + "sa"] = r.reshape(H, W, C).copy()
            r = r + ca(layer_norm(r, w[p + "norm2.weight"], w[p + "norm2.bias"]))
            out[p + "ca"] = r.reshape(H, W, C).copy()
            r = r + self._ffn(p, layer_norm(r, w[p + "norm3.weight"], w[p + "norm3.bias"]))
            out[p + "out"] = r.reshape(H, W, C).copy()
        out["y"] = r
        return out


def make_block(cfg, weights, context_tokens=None, gn_mode=GN_CORRECTED, context=CTX_DISPLACED):
    if cfg.get("batch", 1) > 1:
        return GuidanceBatch(cfg, weights, context_tokens, gn_mode, context)
    if cfg["block"] == "res_attn":
        return ResAttnBlock(cfg, weights, gn_mode, context)
    return SDXLStage(cfg, weights, context_tokens, gn_mode, context)


class GuidanceBatch:
    """B images through the same layer (or stage) step: the classifier-free-guidance
    batch, a conditional and an unconditional branch at guidance scale 5 ([CSDN]
    Implementation details; [README] Benchmarks, --guidance_scale).  The multi-GPU
    original may send the two branches to separate device groups unless
    --no_split_batch is given ([README] Benchmarks, Latency); either way every image
    is its own displaced-patch step -- its own GroupNorm statistics, halo rows and K/V
    context, and for the transformer stage its own text context -- and the images
    share only the weights and the step schedule.  x is [B, H, W, C]; contexts is
    [B, ctx_len, ctx_dim] (transformer stage) or None.  Every returned array gains a
    leading image axis."""

    def __init__(self, cfg, weights, contexts=None, gn_mode=GN_CORRECTED, context=CTX_DISPLACED):
        one = dict(cfg, batch=1)
        self.blocks = [make_block(one, weights, None if contexts is None else contexts[b], gn_mode, context)
                       for b in range(cfg["batch"])]

    def step(self, x, step, is_sync, **kw):
        outs = [blk.step(xb, step, is_sync, **kw) for blk, xb in zip(self.blocks, x)]
        return {k: np.stack([o[k] for o in outs]) if isinstance(outs[0][k], np.ndarray) else [o[k] for o in outs]
                for k in outs[0]}
