"""A CPU stand-in for one patch-parallel rank, for the host-side tests of the exchange.

It keeps the library's buffers in the library's layouts (fp32 storage, as bytes):
k, v [2][heads][L][64], mom1, mom2 [2][N][G][2] (mean, variance), slab [2][N][R+2][W][C]
and y [L][C], with the same parity alternation, and computes a step from those buffers
with the oracle's pieces -- the whole map on a synchronous step, only its patch range on a
displaced step, reading every other patch's context from the buffers the exchange filled.
patch_diffusion_unet_b200.patch_parallel's exchange runs on it unchanged, so a two-rank
gloo run checks the partition, the gather layouts, the halo rows at the range ends and the
step-to-step ordering against the single-process oracle.  Test infrastructure only.
"""
import contextlib

import numpy as np
import torch

import oracle
from patch_diffusion_unet_b200.patch_parallel import partition


class OracleRank:
    def __init__(self, cfg, weights, rank, world, gn_mode=oracle.GN_CORRECTED):
        self.cfg, self.rank, self.world, self.gn_mode = cfg, rank, world, gn_mode
        self.p0, self.p1 = partition(cfg["n_patches"], world, rank)
        H, W, C, N, G, heads = (cfg[k] for k in ("H", "W", "C", "n_patches", "gn_groups", "heads"))
        self.R, self.L = H // N, H * W
        self.w = {k: np.asarray(v, np.float64) for k, v in weights.items()}
        z = lambda n: [torch.zeros(n, dtype=torch.float32) for _ in range(2)]  # noqa: E731
        self.k, self.v = z(heads * self.L * 64), z(heads * self.L * 64)
        self.mom1, self.mom2 = z(N * G * 2), z(N * G * 2)
        self.slab = z(N * (self.R + 2) * W * C)
        self.y = torch.zeros(self.L * C, dtype=torch.float32)

    # ---- what the exchange sees
    def buffer(self, name, parity):
        t = self.y if name == "y" else getattr(self, name)[parity]
        return t.view(torch.uint8)

    def stream_context(self):
        return contextlib.nullcontext()

    # ---- views in the layouts
    def _slab(self, par):
        c = self.cfg
        return self.slab[par].view(c["n_patches"], self.R + 2, c["W"], c["C"])

    def _kv(self, buf, par):
        c = self.cfg
        return buf[par].view(c["heads"], self.L, 64)

    def _gn(self, x_rows, mom, par, patches, is_sync, gamma, beta, silu):
        """GroupNorm of the given patches of x (rows of the whole map) from the buffers."""
        c = self.cfg
        N, G = c["n_patches"], c["gn_groups"]
        bounds = oracle.patch_bounds(c["H"], N)
        m = mom[par].view(N, G, 2)
        fresh = np.zeros((N, G, 2))
        for p in patches:
            r0, r1 = bounds[p]
            fresh[p] = oracle.group_moments(x_rows[r0:r1], G)
            m[p] = torch.from_numpy(np.stack([fresh[p][:, 0], fresh[p][:, 1] - fresh[p][:, 0] ** 2], -1))
        stale = None
        if not is_sync:
            s = mom[par ^ 1].view(N, G, 2).double().numpy()
            stale = np.stack([s[..., 0], s[..., 1] + s[..., 0] ** 2], -1)     # back to (E[x], E[x^2])
        mu, var = oracle.merge_moments(fresh, stale, is_sync, self.gn_mode)
        out = {}
        for p in patches:
            r0, r1 = bounds[p]
            y = oracle.normalize(x_rows[r0:r1], mu[p], var[p], gamma, beta, c["gn_eps"])
            out[p] = oracle.silu(y) if silu else y
        return out

    def compute(self, x, step, is_sync):
        c, w = self.cfg, self.w
        N, W, C, heads = c["n_patches"], c["W"], c["C"], c["heads"]
        R, L = self.R, self.L
        par = step & 1
        x = np.asarray(x, np.float64)
        patches = range(N) if is_sync else range(self.p0, self.p1)
        slab, prev = self._slab(par), self._slab(par ^ 1)
        y1 = self._gn(x, self.mom1, par, patches, is_sync, w["gn1.weight"], w["gn1.bias"], True)
        for p in patches:
            slab[p, 1:R + 1] = torch.from_numpy(y1[p])
        # halo rows: image edges zero; this step's neighbour rows when synchronous; on a
        # displaced step the previous step's rows inside the range, the exchange's at its ends
        for p in patches:
            if p == 0:
                slab[p, 0] = 0
            elif is_sync:
                slab[p, 0] = slab[p - 1, R]
            elif p > self.p0:
                slab[p, 0] = prev[p - 1, R]
            if p == N - 1:
                slab[p, R + 1] = 0
            elif is_sync:
                slab[p, R + 1] = slab[p + 1, 1]
            elif p < self.p1 - 1:
                slab[p, R + 1] = prev[p + 1, 1]
        h = np.zeros((c["H"], W, C))
        for p in patches:
            h[p * R:(p + 1) * R] = oracle.conv3x3_rows(slab[p].double().numpy(), w["conv1.weight"], w["conv1.bias"])
        t = self._gn(h, self.mom2, par, patches, is_sync, w["gn2.weight"], w["gn2.bias"], False)
        kc, vc = self._kv(self.k, par), self._kv(self.v, par)
        ks, vs = self._kv(self.k, par ^ 1), self._kv(self.v, par ^ 1)
        q = {}
        Lp = R * W
        for p in patches:
            tok = t[p].reshape(Lp, C)
            q[p] = tok @ w["attn.to_q.weight"].T
            kk, vv = tok @ w["attn.to_k.weight"].T, tok @ w["attn.to_v.weight"].T
            for hd in range(heads):
                kc[hd, p * Lp:(p + 1) * Lp] = torch.from_numpy(kk[:, hd * 64:(hd + 1) * 64])
                vc[hd, p * Lp:(p + 1) * Lp] = torch.from_numpy(vv[:, hd * 64:(hd + 1) * 64])
        y = self.y.view(L, C)
        for p in patches:
            a, b = p * Lp, (p + 1) * Lp
            o = np.zeros((Lp, C))
            for hd in range(heads):
                if is_sync:
                    K, V = kc[hd].double().numpy(), vc[hd].double().numpy()
                else:
                    K, V = ks[hd].double().numpy().copy(), vs[hd].double().numpy().copy()
                    K[a:b], V[a:b] = kc[hd, a:b].double().numpy(), vc[hd, a:b].double().numpy()
                o[:, hd * 64:(hd + 1) * 64] = oracle.softmax_attention(q[p][:, hd * 64:(hd + 1) * 64], K, V, 1.0 / 8.0)
            y[a:b] = torch.from_numpy(o @ w["attn.to_out.weight"].T + w["attn.to_out.bias"])

    def output(self):
        return self.y.view(self.L, self.cfg["C"]).double().numpy()
