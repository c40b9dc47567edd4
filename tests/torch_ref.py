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
