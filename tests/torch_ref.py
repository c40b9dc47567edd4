"""Full-image (unpatched) layers written with PyTorch's own CPU fp64 library routines.

Used only by the oracle's pins: a synchronous displaced-patch step, an N=1
step, or a step whose stale context equals the fresh one must reproduce the
single-device layer, "the original diffusion model running on one device"
("DistriFusion" project README, Overview (a) and (c)).
"""
import numpy as np
import torch
import torch.nn.functional as F


def _t(a):
    return torch.from_numpy(np.asarray(a, np.float64))


def _nchw(x):
    return _t(x).permute(2, 0, 1)[None]


def _nhwc(X):
    return X[0].permute(1, 2, 0).numpy()


def _mha(tok, wq, wk, wv, wo, bo, heads, ctx=None):
    ctx = tok if ctx is None else ctx
    L, C = tok.shape
    d = C // heads
    q = F.linear(tok, _t(wq)).view(L, heads, d).transpose(0, 1)
    k = F.linear(ctx, _t(wk)).view(ctx.shape[0], heads, d).transpose(0, 1)
    v = F.linear(ctx, _t(wv)).view(ctx.shape[0], heads, d).transpose(0, 1)
    o = F.scaled_dot_product_attention(q, k, v).transpose(0, 1).reshape(L, C)
    return F.linear(o, _t(wo), _t(bo)), o


def res_attn_full(x, w, cfg):
    """GN+SiLU -> conv3x3(pad 1) -> GN -> MHA(Q,K,V no bias; out with bias) on a whole map."""
    G, eps = cfg["gn_groups"], cfg["gn_eps"]
    X = _nchw(x)
    y1 = F.silu(F.group_norm(X, G, _t(w["gn1.weight"]), _t(w["gn1.bias"]), eps))
    h = F.conv2d(y1, _t(w["conv1.weight"]), _t(w["conv1.bias"]), padding=1)
    t = F.group_norm(h, G, _t(w["gn2.weight"]), _t(w["gn2.bias"]), eps)
    H, W, C = x.shape
    tok = t[0].permute(1, 2, 0).reshape(H * W, C)
    y, o = _mha(tok, w["attn.to_q.weight"], w["attn.to_k.weight"], w["attn.to_v.weight"],
                w["attn.to_out.weight"], w["attn.to_out.bias"], cfg["heads"])
    return dict(y=y.numpy(), y1=_nhwc(y1), h=_nhwc(h), t=_nhwc(t), o=o.numpy())


def sdxl_stage_full(x, w, ctx, cfg):
    """ResNet block + transformer blocks (pre-LN SA, CA, GEGLU FFN with exact GELU) on a whole map."""
    G, eps, C = cfg["gn_groups"], cfg["gn_eps"], cfg["C"]
    X = _nchw(x)
    h = F.conv2d(F.silu(F.group_norm(X, G, _t(w["resnet.norm1.weight"]), _t(w["resnet.norm1.bias"]), eps)),
                 _t(w["resnet.conv1.weight"]), _t(w["resnet.conv1.bias"]), padding=1)
    h = F.conv2d(F.silu(F.group_norm(h, G, _t(w["resnet.norm2.weight"]), _t(w["resnet.norm2.bias"]), eps)),
                 _t(w["resnet.conv2.weight"]), _t(w["resnet.conv2.bias"]), padding=1)
    H, W, _ = x.shape
    r = (X + h)[0].permute(1, 2, 0).reshape(H * W, C)
    c = _t(ctx)
    for b in range(cfg["n_xformer"]):
        p = f"xf{b}."

        def ln(u, n):
            return F.layer_norm(u, (C,), _t(w[p + n + ".weight"]), _t(w[p + n + ".bias"]), 1e-5)

        r = r + _mha(ln(r, "norm1"), w[p + "attn1.to_q.weight"], w[p + "attn1.to_k.weight"],
                     w[p + "attn1.to_v.weight"], w[p + "attn1.to_out.weight"],
                     w[p + "attn1.to_out.bias"], cfg["heads"])[0]
        r = r + _mha(ln(r, "norm2"), w[p + "attn2.to_q.weight"], w[p + "attn2.to_k.weight"],
                     w[p + "attn2.to_v.weight"], w[p + "attn2.to_out.weight"],
                     w[p + "attn2.to_out.bias"], cfg["heads"], ctx=c)[0]
        hg = F.linear(ln(r, "norm3"), _t(w[p + "ff.proj.weight"]), _t(w[p + "ff.proj.bias"]))
        a, gate = hg.chunk(2, dim=-1)
        r = r + F.linear(a * F.gelu(gate), _t(w[p + "ff.out.weight"]), _t(w[p + "ff.out.bias"]))
    return dict(y=r.numpy())


# ---------------------------------------------------------------- batched (guidance batch)
# The same layers on a batch [B, H, W, C] with PyTorch's batched routines: group_norm
# takes its statistics per sample, conv2d runs per sample, and scaled_dot_product_attention
# attends within each batch element -- so these pin that a batch of images never mixes.

def _mha_batched(tok, wq, wk, wv, wo, bo, heads, ctx=None):
    ctx = tok if ctx is None else ctx
    B, L, C = tok.shape
    d = C // heads

    def split(u):
        return u.view(B, u.shape[1], heads, d).transpose(1, 2)

    q, k, v = split(F.linear(tok, _t(wq))), split(F.linear(ctx, _t(wk))), split(F.linear(ctx, _t(wv)))
    o = F.scaled_dot_product_attention(q, k, v).transpose(1, 2).reshape(B, L, C)
    return F.linear(o, _t(wo), _t(bo)), o


def res_attn_full_batched(xs, w, cfg):
    """res_attn_full on a batch xs [B, H, W, C]; arrays come back with a leading batch axis."""
    G, eps = cfg["gn_groups"], cfg["gn_eps"]
    B, H, W, C = xs.shape
    X = _t(xs).permute(0, 3, 1, 2)
    y1 = F.silu(F.group_norm(X, G, _t(w["gn1.weight"]), _t(w["gn1.bias"]), eps))
    h = F.conv2d(y1, _t(w["conv1.weight"]), _t(w["conv1.bias"]), padding=1)
    t = F.group_norm(h, G, _t(w["gn2.weight"]), _t(w["gn2.bias"]), eps)
    tok = t.permute(0, 2, 3, 1).reshape(B, H * W, C)
    y, o = _mha_batched(tok, w["attn.to_q.weight"], w["attn.to_k.weight"], w["attn.to_v.weight"],
                        w["attn.to_out.weight"], w["attn.to_out.bias"], cfg["heads"])
    nhwc = lambda a: a.permute(0, 2, 3, 1).numpy()  # noqa: E731
    return dict(y=y.numpy(), y1=nhwc(y1), h=nhwc(h), t=nhwc(t), o=o.numpy())


def sdxl_stage_full_batched(xs, w, ctxs, cfg):
    """sdxl_stage_full on a batch xs [B, H, W, C] with one context per image ctxs [B, T, D]."""
    G, eps, C = cfg["gn_groups"], cfg["gn_eps"], cfg["C"]
    B, H, W, _ = xs.shape
    X = _t(xs).permute(0, 3, 1, 2)
    h = F.conv2d(F.silu(F.group_norm(X, G, _t(w["resnet.norm1.weight"]), _t(w["resnet.norm1.bias"]), eps)),
                 _t(w["resnet.conv1.weight"]), _t(w["resnet.conv1.bias"]), padding=1)
    h = F.conv2d(F.silu(F.group_norm(h, G, _t(w["resnet.norm2.weight"]), _t(w["resnet.norm2.bias"]), eps)),
                 _t(w["resnet.conv2.weight"]), _t(w["resnet.conv2.bias"]), padding=1)
    r = (X + h).permute(0, 2, 3, 1).reshape(B, H * W, C)
    c = _t(ctxs)
    for b in range(cfg["n_xformer"]):
        p = f"xf{b}."

        def ln(u, n):
            return F.layer_norm(u, (C,), _t(w[p + n + ".weight"]), _t(w[p + n + ".bias"]), 1e-5)

        r = r + _mha_batched(ln(r, "norm1"), w[p + "attn1.to_q.weight"], w[p + "attn1.to_k.weight"],
                             w[p + "attn1.to_v.weight"], w[p + "attn1.to_out.weight"],
                             w[p + "attn1.to_out.bias"], cfg["heads"])[0]
        r = r + _mha_batched(ln(r, "norm2"), w[p + "attn2.to_q.weight"], w[p + "attn2.to_k.weight"],
                             w[p + "attn2.to_v.weight"], w[p + "attn2.to_out.weight"],
                             w[p + "attn2.to_out.bias"], cfg["heads"], ctx=c)[0]
        hg = F.linear(ln(r, "norm3"), _t(w[p + "ff.proj.weight"]), _t(w[p + "ff.proj.bias"]))
        a, gate = hg.chunk(2, dim=-1)
        r = r + F.linear(a * F.gelu(gate), _t(w[p + "ff.out.weight"]), _t(w[p + "ff.out.bias"]))
    return dict(y=r.numpy())


# ---------------------------------------------------------------- the multi-level UNet
# The whole (unpatched) network of the UNet workload with PyTorch's routines: strided
# conv2d for the downsampling, interpolate(nearest) for the upsampling, cat for the skips.

def unet_full(x, w, ctx, cfg, tau):
    """Predicted noise of the UNet for latent x [H, W, latent_c] at timestep tau."""
    import math
    G, eps = cfg["gn_groups"], cfg["gn_eps"]
    c0, c1, c2 = cfg["widths"]
    half = c0 // 2
    f = torch.exp(-math.log(10000.0) * torch.arange(half, dtype=torch.float64) / half)
    e = torch.cat([torch.cos(float(tau) * f), torch.sin(float(tau) * f)])
    temb = F.linear(F.silu(F.linear(e, _t(w["time_embedding.linear_1.weight"]), _t(w["time_embedding.linear_1.bias"]))),
                    _t(w["time_embedding.linear_2.weight"]), _t(w["time_embedding.linear_2.bias"]))
    ta = F.silu(temb)
    c = _t(ctx)

    def gn_silu(h, n):
        return F.silu(F.group_norm(h, G, _t(w[n + ".weight"]), _t(w[n + ".bias"]), eps))

    def conv(h, n, stride=1):
        return F.conv2d(h, _t(w[n + ".weight"]), _t(w[n + ".bias"]), stride=stride, padding=1)

    def resnet(h, p):
        y = conv(gn_silu(h, p + "norm1"), p + "conv1") + \
            F.linear(ta, _t(w[p + "time_emb_proj.weight"]), _t(w[p + "time_emb_proj.bias"]))[None, :, None, None]
        y = conv(gn_silu(y, p + "norm2"), p + "conv2")
        if p + "conv_shortcut.weight" in w:
            h = F.conv2d(h, _t(w[p + "conv_shortcut.weight"])[:, :, None, None], _t(w[p + "conv_shortcut.bias"]))
        return h + y

    def xf(h, p):
        _, C, H, W = h.shape
        r = h[0].permute(1, 2, 0).reshape(H * W, C)

        def ln(u, n):
            return F.layer_norm(u, (C,), _t(w[p + n + ".weight"]), _t(w[p + n + ".bias"]), 1e-5)

        r = r + _mha(ln(r, "norm1"), w[p + "attn1.to_q.weight"], w[p + "attn1.to_k.weight"], w[p + "attn1.to_v.weight"],
                     w[p + "attn1.to_out.weight"], w[p + "attn1.to_out.bias"], C // 64)[0]
        r = r + _mha(ln(r, "norm2"), w[p + "attn2.to_q.weight"], w[p + "attn2.to_k.weight"], w[p + "attn2.to_v.weight"],
                     w[p + "attn2.to_out.weight"], w[p + "attn2.to_out.bias"], C // 64, ctx=c)[0]
        hg = F.linear(ln(r, "norm3"), _t(w[p + "ff.proj.weight"]), _t(w[p + "ff.proj.bias"]))
        a, gate = hg.chunk(2, dim=-1)
        r = r + F.linear(a * F.gelu(gate), _t(w[p + "ff.out.weight"]), _t(w[p + "ff.out.bias"]))
        return r.reshape(H, W, C).permute(2, 0, 1)[None]

    up = lambda h: F.interpolate(h, scale_factor=2, mode="nearest")  # noqa: E731
    h = conv(_nchw(x), "conv_in")
    s0 = h = resnet(h, "down0.resnet.")
    h = conv(h, "down0.downsample", stride=2)
    s1 = h = xf(resnet(h, "down1.resnet."), "down1.xf.")
    h = conv(h, "down1.downsample", stride=2)
    mid = h = xf(resnet(h, "down2.resnet."), "down2.xf.")
    h = xf(resnet(torch.cat([conv(up(h), "up1.upsample"), s1], 1), "up1.resnet."), "up1.xf.")
    h = resnet(torch.cat([conv(up(h), "up0.upsample"), s0], 1), "up0.resnet.")
    out = conv(gn_silu(h, "norm_out"), "conv_out")
    return dict(eps=_nhwc(out), mid=_nhwc(mid), s0=_nhwc(s0), s1=_nhwc(s1), up0=_nhwc(h))
