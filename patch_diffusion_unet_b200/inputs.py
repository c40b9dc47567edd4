"""Seeded synthetic inputs for the displaced-patch layer step.

This module draws random numbers and rounds them to the workload's storage
type; it holds none of the method's arithmetic.  Both the CPU oracle (through
the tests and the benchmark's CPU leg) and the CUDA path consume exactly the
arrays produced here.

Recipe (fixed, seed 0 unless stated):
  rng = numpy.random.default_rng(seed); fp64 standard normals are drawn in this
  order: every drawn weight in declaration order (``weight_specs``), then the
  cross-attention context (transformer stage only), then x_0, then the noise
  e_t for t = 1, 2, ...  Weights and biases are 0.02 * N(0, 1).  Norm scales
  are 1 and norm shifts 0 (PyTorch's default init; not drawn).  The layer
  input drifts as an AR(1) process, x_t = 0.95 x_{t-1} + 0.05 e_t, evaluated
  in fp64.  Every array handed out is cast fp64 -> fp32 -> storage type with
  round-to-nearest-even, and returned as float32 whose values are exactly
  representable in the storage type.

  A batch of B images (workload key "batch", the classifier-free-guidance batch):
  image 0 is the single-image workload above, unchanged; image b >= 1 draws its
  own context (transformer stage) and then its x_0, e_1, e_2, ... from
  numpy.random.default_rng([seed, b]).  The weights are image 0's.  x(t) is then
  [B, H, W, C] and the context [B, ctx_len, ctx_dim].

Stand-in for the pages' workload: SDXL latents of COCO-caption prompts
("DistriFusion: Distributed Parallel Inference for High-Resolution Diffusion
Models" README, Benchmarks / COCO quality) are not available; these synthetic
maps have the same shapes as one SDXL UNet level.
"""
import numpy as np
import torch

RHO = 0.95
NOISE = 0.05
WEIGHT_STD = 0.02


def round_to(a, dtype):
    """Cast to fp32, then (for "bf16") round-to-nearest-even to bfloat16; return fp32 values."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "f32":
        return a32
    if dtype == "bf16":
        return torch.from_numpy(a32).to(torch.bfloat16).to(torch.float32).numpy()
    raise ValueError(f"unknown dtype {dtype!r}")


def to_torch(a32, dtype):
    """Host torch tensor in the storage type (lossless for arrays from this module)."""
    t = torch.from_numpy(np.ascontiguousarray(a32, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def fixed_specs(cfg):
    """Norm affine parameters (not drawn): list of (name, shape, fill)."""
    if cfg["block"] == "unet":
        return unet_fixed_specs(cfg)
    C = cfg["C"]
    out = []
    if cfg["block"] == "res_attn":
        for n in ("gn1", "gn2"):
            out += [(f"{n}.weight", (C,), 1.0), (f"{n}.bias", (C,), 0.0)]
    else:
        for n in ("resnet.norm1", "resnet.norm2"):
            out += [(f"{n}.weight", (C,), 1.0), (f"{n}.bias", (C,), 0.0)]
        for b in range(cfg["n_xformer"]):
            for n in ("norm1", "norm2", "norm3"):
                out += [(f"xf{b}.{n}.weight", (C,), 1.0), (f"xf{b}.{n}.bias", (C,), 0.0)]
    return out


def weight_specs(cfg):
    """Drawn weights in declaration order: list of (name, shape), PyTorch layouts
    (conv [Cout, Cin, 3, 3], linear [out, in])."""
    if cfg["block"] == "unet":
        return unet_weight_specs(cfg)
    C = cfg["C"]
    if cfg["block"] == "res_attn":
        return [
            ("conv1.weight", (C, C, 3, 3)), ("conv1.bias", (C,)),
            ("attn.to_q.weight", (C, C)), ("attn.to_k.weight", (C, C)),
            ("attn.to_v.weight", (C, C)), ("attn.to_out.weight", (C, C)),
            ("attn.to_out.bias", (C,)),
        ]
    D, F = cfg["ctx_dim"], cfg["ffn_inner"]
    specs = [
        ("resnet.conv1.weight", (C, C, 3, 3)), ("resnet.conv1.bias", (C,)),
        ("resnet.conv2.weight", (C, C, 3, 3)), ("resnet.conv2.bias", (C,)),
    ]
    for b in range(cfg["n_xformer"]):
        p = f"xf{b}."
        specs += [
            (p + "attn1.to_q.weight", (C, C)), (p + "attn1.to_k.weight", (C, C)),
            (p + "attn1.to_v.weight", (C, C)), (p + "attn1.to_out.weight", (C, C)),
            (p + "attn1.to_out.bias", (C,)),
            (p + "attn2.to_q.weight", (C, C)), (p + "attn2.to_k.weight", (C, D)),
            (p + "attn2.to_v.weight", (C, D)), (p + "attn2.to_out.weight", (C, C)),
            (p + "attn2.to_out.bias", (C,)),
            (p + "ff.proj.weight", (2 * F, C)), (p + "ff.proj.bias", (2 * F,)),
            (p + "ff.out.weight", (C, F)), (p + "ff.out.bias", (C,)),
        ]
    return specs


def unet_weight_specs(cfg):
    """Drawn weights of the multi-level UNet (name, shape) in declaration order, PyTorch
    layouts: timestep MLP, conv_in, per level a ResNet block (1x1 shortcut when the width
    changes), transformer blocks at the two lower levels, down / up convs, conv_out."""
    c0, c1, c2 = cfg["widths"]
    D, lat = cfg["ctx_dim"], cfg["latent_c"]
    specs = [("time_embedding.linear_1.weight", (4 * c0, c0)), ("time_embedding.linear_1.bias", (4 * c0,)),
             ("time_embedding.linear_2.weight", (4 * c0, 4 * c0)), ("time_embedding.linear_2.bias", (4 * c0,)),
             ("conv_in.weight", (c0, lat, 3, 3)), ("conv_in.bias", (c0,))]

    def resnet(p, ci, co):
        s = [(p + "conv1.weight", (co, ci, 3, 3)), (p + "conv1.bias", (co,)),
             (p + "time_emb_proj.weight", (co, 4 * c0)), (p + "time_emb_proj.bias", (co,)),
             (p + "conv2.weight", (co, co, 3, 3)), (p + "conv2.bias", (co,))]
        if ci != co:
            s += [(p + "conv_shortcut.weight", (co, ci)), (p + "conv_shortcut.bias", (co,))]
        return s

    def xf(p, c):
        F = 4 * c
        return [(p + "attn1.to_q.weight", (c, c)), (p + "attn1.to_k.weight", (c, c)), (p + "attn1.to_v.weight", (c, c)),
                (p + "attn1.to_out.weight", (c, c)), (p + "attn1.to_out.bias", (c,)),
                (p + "attn2.to_q.weight", (c, c)), (p + "attn2.to_k.weight", (c, D)), (p + "attn2.to_v.weight", (c, D)),
                (p + "attn2.to_out.weight", (c, c)), (p + "attn2.to_out.bias", (c,)),
                (p + "ff.proj.weight", (2 * F, c)), (p + "ff.proj.bias", (2 * F,)),
                (p + "ff.out.weight", (c, F)), (p + "ff.out.bias", (c,))]

    specs += resnet("down0.resnet.", c0, c0)
    specs += [("down0.downsample.weight", (c0, c0, 3, 3)), ("down0.downsample.bias", (c0,))]
    specs += resnet("down1.resnet.", c0, c1) + xf("down1.xf.", c1)
    specs += [("down1.downsample.weight", (c1, c1, 3, 3)), ("down1.downsample.bias", (c1,))]
    specs += resnet("down2.resnet.", c1, c2) + xf("down2.xf.", c2)
    specs += [("up1.upsample.weight", (c2, c2, 3, 3)), ("up1.upsample.bias", (c2,))]
    specs += resnet("up1.resnet.", c2 + c1, c1) + xf("up1.xf.", c1)
    specs += [("up0.upsample.weight", (c1, c1, 3, 3)), ("up0.upsample.bias", (c1,))]
    specs += resnet("up0.resnet.", c1 + c0, c0)
    specs += [("conv_out.weight", (lat, c0, 3, 3)), ("conv_out.bias", (lat,))]
    return specs


def unet_fixed_specs(cfg):
    """Norm scales / shifts of the UNet (name, shape, fill): 1 and 0, not drawn."""
    c0, c1, c2 = cfg["widths"]
    out = []
    for p, ci, co in (("down0.resnet.", c0, c0), ("down1.resnet.", c0, c1), ("down2.resnet.", c1, c2),
                      ("up1.resnet.", c2 + c1, c1), ("up0.resnet.", c1 + c0, c0)):
        out += [(p + "norm1.weight", (ci,), 1.0), (p + "norm1.bias", (ci,), 0.0),
                (p + "norm2.weight", (co,), 1.0), (p + "norm2.bias", (co,), 0.0)]
    for p, c in (("down1.xf.", c1), ("down2.xf.", c2), ("up1.xf.", c1)):
        for n in ("norm1", "norm2", "norm3"):
            out += [(p + n + ".weight", (c,), 1.0), (p + n + ".bias", (c,), 0.0)]
    out += [("norm_out.weight", (c0,), 1.0), ("norm_out.bias", (c0,), 0.0)]
    return out


class SyntheticWorkload:
    """Weights, context and the drifting layer inputs x_0, x_1, ... of one workload.

    ``weight_scale`` multiplies chosen drawn weights after drawing (e.g. a larger
    scale on to_q/to_k gives peaked attention); ``random_affine`` replaces the norm
    scales/shifts by 1 + 0.1 N(0,1) / 0.1 N(0,1) drawn from a separate stream
    (seed + 1), leaving the main stream untouched.
    """

    def __init__(self, cfg, seed=0, weight_scale=None, random_affine=False):
        self.cfg = cfg
        self.dtype = cfg["dtype"]
        self.rng = np.random.default_rng(seed)
        self.weights = {}
        scale = weight_scale or {}
        for name, shape in weight_specs(cfg):
            w = self.rng.standard_normal(shape) * WEIGHT_STD * scale.get(name, 1.0)
            self.weights[name] = round_to(w, self.dtype)
        arng = np.random.default_rng(seed + 1)
        for name, shape, fill in fixed_specs(cfg):
            if random_affine:
                v = (1.0 if fill == 1.0 else 0.0) + 0.1 * arng.standard_normal(shape)
            else:
                v = np.full(shape, fill)
            self.weights[name] = round_to(v, self.dtype)
        self.batch = cfg.get("batch", 1)
        # image b >= 1 of a batch: its own stream for its context and its inputs
        self.rngs = [self.rng] + [np.random.default_rng([seed, b]) for b in range(1, self.batch)]
        self.context = None
        if cfg["block"] in ("sdxl_stage", "unet"):
            ctx = [round_to(r.standard_normal((cfg["ctx_len"], cfg["ctx_dim"])), self.dtype) for r in self.rngs]
            self.context = ctx[0] if self.batch == 1 else np.stack(ctx)
        self._state = None   # fp64 x_t, one per image
        self._t = -1

    def latent(self):
        """The UNet workload's starting latent x_T ~ N(0, 1), [H, W, latent_c] (drawn after the
        context from the main stream; the DDIM loop evolves it from there)."""
        if not hasattr(self, "_latent"):
            shape = (self.cfg["H"], self.cfg["W"], self.cfg["latent_c"])
            self._latent = round_to(self.rng.standard_normal(shape), self.dtype)
        return self._latent

    def x(self, t):
        """Layer input of step t (must be requested in order 0, 1, 2, ...; repeats allowed)."""
        if t == self._t:
            return self._cur
        if t != self._t + 1:
            raise ValueError(f"inputs are drawn sequentially: asked for step {t} after {self._t}")
        shape = (self.cfg["H"], self.cfg["W"], self.cfg["C"])
        if t == 0:
            self._state = [r.standard_normal(shape) for r in self.rngs]
        else:
            self._state = [RHO * s + NOISE * r.standard_normal(shape) for s, r in zip(self._state, self.rngs)]
        self._t = t
        cur = [round_to(s, self.dtype) for s in self._state]
        self._cur = cur[0] if self.batch == 1 else np.stack(cur)
        return self._cur

    def schedule(self):
        """(step, is_sync) for the whole run: the first n_sync steps are synchronous."""
        return [(t, int(t < self.cfg["n_sync"])) for t in range(self.cfg["steps"])]
