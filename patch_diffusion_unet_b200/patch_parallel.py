"""Patch parallelism across GPUs: one process per GPU, each computing its own row patches.

The pages' system runs one patch per device ("DistriFusion" project README, Overview (c)):
every device computes its own rows fresh and takes the other patches' activations of the
previous step as context, exchanged asynchronously; the exchange is an AllGather (paper
reading blog, Ablation: patch parallelism gathers rather than all-reduces).  Here rank r
of `world` owns the contiguous patch range [r N/world, (r+1) N/world) of the layer's N
patches and holds a library handle for the whole map:

* a synchronous step runs the whole map on every rank (dfp_step; each rank holds the full
  latent), so every rank's buffers are complete afterwards;
* a displaced step runs only the rank's patches (dfp_step_patches) -- their GroupNorm
  merges read the previous step's moments of every patch, their conv reads the previous
  step's boundary rows of the neighbouring patches, their attention the previous step's
  K/V of every other patch -- and is followed by the exchange: in-place all-gathers of the
  step's K/V rows (per head), GroupNorm moments, the ranks' boundary rows of the conv input
  and the output rows, so every rank's buffers hold the whole map again and the next
  displaced step finds its stale context in place.

The exchange only moves bytes between library-owned buffers (dfp_context_buffer); the
arithmetic of the step runs in the library's kernels.  Two transports carry the
all-gathers: DistTransport (torch.distributed, NCCL over NVLink on GPUs, gloo on the host)
and LocalTransport, which emulates the ranks of one process by copies (one GPU standing in
for several, with no kernel of one rank waiting on another's).
"""
import ctypes

import torch


def partition(n_patches, world, rank):
    """The rank's patch range [p0, p1) (contiguous, equal shares)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    if n_patches % world:
        raise ValueError(f"{n_patches} patches do not divide among {world} ranks")
    per = n_patches // world
    return rank * per, (rank + 1) * per


class _DeviceBytes:
    """A raw device range seen as a torch uint8 tensor (no copy, library-owned memory)."""

    def __init__(self, ptr, nbytes):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1", "data": (ptr, False),
                                         "version": 3, "strides": None}


def layout(cfg):
    """Byte sizes of the exchanged buffers of one image: (element size, tokens per patch,
    rows per patch)."""
    e = 2 if cfg["dtype"] == "bf16" else 4
    R = cfg["H"] // cfg["n_patches"]
    return e, R * cfg["W"], R


def gathers(cfg, bufs, parity, rank, world):
    """The in-place all-gathers after a displaced step of `parity`: a list of
    (full, own) uint8 tensors, `full` the whole gathered range (world equal chunks in rank
    order) and `own` this rank's chunk of it.  bufs(name, parity) -> uint8 tensor of the
    library buffer.  The boundary rows travel separately (boundary_rows)."""
    e, Lp, _ = layout(cfg)
    N, C, G, heads = cfg["n_patches"], cfg["C"], cfg["gn_groups"], cfg["heads"]
    per = N // world
    L = N * Lp
    out = []

    def add(full, chunk):
        out.append((full, full[rank * chunk:(rank + 1) * chunk]))

    for name in ("k", "v"):                        # [heads][L][64]: one gather per head
        b = bufs(name, parity)
        head = L * 64 * e
        for h in range(heads):
            add(b[h * head:(h + 1) * head], per * Lp * 64 * e)
    for name in ("mom1", "mom2"):                  # [N][G][2] fp32
        add(bufs(name, parity), per * G * 2 * 4)
    add(bufs("y", parity), per * Lp * C * e)       # [L][C]
    return out


def boundary_rows(cfg, bufs, parity, rank, world):
    """(pack, recv, fill) for the boundary rows of the conv input after a step of `parity`.
    recv, [world][2][W*C*e] bytes, receives every rank's first patch's first row and last
    patch's last row; pack() writes this rank's pair into its own chunk of recv (the input
    of the in-place gather); fill() then writes the neighbouring ranks' rows into this
    rank's halo rows at its range ends in the other parity's slab, where the next step's
    conv reads them (boundaries inside the range are copied by that step's GroupNorm
    kernel itself)."""
    e, _, R = layout(cfg)
    W, C = cfg["W"], cfg["C"]
    per = cfg["n_patches"] // world
    row = W * C * e
    patch = (R + 2) * row
    cur, nxt = bufs("slab", parity), bufs("slab", parity ^ 1)
    recv = torch.empty(world * 2 * row, dtype=torch.uint8, device=cur.device)

    def pack(r=rank):
        a, b = r * per, (r + 1) * per
        recv[r * 2 * row:r * 2 * row + row].copy_(cur[a * patch + row:a * patch + 2 * row])       # patch a, row 1
        recv[r * 2 * row + row:(r + 1) * 2 * row].copy_(cur[(b - 1) * patch + R * row:
                                                            (b - 1) * patch + (R + 1) * row])     # patch b-1, row R

    def fill():
        p0, p1 = rank * per, (rank + 1) * per
        if rank > 0:          # top halo of p0 <- last row of patch p0-1 (the previous rank's)
            nxt[p0 * patch:p0 * patch + row].copy_(recv[(rank - 1) * 2 * row + row:rank * 2 * row])
        if rank < world - 1:  # bottom halo of p1-1 <- first row of patch p1 (the next rank's)
            o = (p1 - 1) * patch + (R + 1) * row
            nxt[o:o + row].copy_(recv[(rank + 1) * 2 * row:(rank + 1) * 2 * row + row])
    return pack, recv, fill


def halo_from_local(cfg, bufs, parity, rank, world):
    """After a synchronous step every buffer is complete on every rank: the halo rows at
    the range ends of the other parity's slab are filled from this rank's own copy."""
    pack, _, fill = boundary_rows(cfg, bufs, parity, rank, world)
    for r in range(world):      # every rank's boundary pair, read from the local slab
        pack(r)
    fill()


class DistTransport:
    """All-gathers through torch.distributed (one rank per process)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group

    def all_gather(self, pairs_per_rank):
        (pairs,) = pairs_per_rank
        for full, own in pairs:
            self.dist.all_gather_into_tensor(full, own, group=self.group)


class LocalTransport:
    """All-gathers among ranks emulated in one process: rank r's chunk is copied into every
    other rank's buffer (the transport of one GPU standing in for several)."""

    def all_gather(self, pairs_per_rank):
        world = len(pairs_per_rank)
        for i in range(len(pairs_per_rank[0])):
            for r in range(world):
                own = pairs_per_rank[r][i][1]
                for q in range(world):
                    if q != r:
                        full = pairs_per_rank[q][i][0]
                        n = own.numel()
                        full[r * n:(r + 1) * n].copy_(own)


class PatchParallelLayer:
    """Rank `rank` of a patch-parallel displaced-patch layer (one library handle for the
    whole map; see the module docstring)."""

    def __init__(self, cfg, rank, world, stream=None, gn_mode=0, context=0):
        from . import dfp
        self.dfp = dfp
        self.cfg, self.rank, self.world = cfg, rank, world
        self.p0, self.p1 = partition(cfg["n_patches"], world, rank)
        self.blk = dfp.DisplacedPatchBlock(cfg, stream=stream, gn_mode=gn_mode, context=context)
        self._views = {}

    def load_weights(self, weights):
        self.blk.load_weights(weights)

    def buffer(self, name, parity):
        """A library buffer as a uint8 device tensor (no copy)."""
        key = (name, parity)
        if key not in self._views:
            ptr, nbytes = ctypes.c_void_p(), ctypes.c_longlong()
            st = self.dfp.LIB.dfp_context_buffer(self.blk.h, name.encode(), parity, ctypes.byref(ptr),
                                                  ctypes.byref(nbytes))
            self.blk._check(st)
            self._views[key] = torch.as_tensor(_DeviceBytes(ptr.value, nbytes.value), device="cuda")
        return self._views[key]

    def compute(self, x, step, is_sync):
        """This rank's part of the step: the whole map when synchronous (or world == 1),
        its patch range otherwise."""
        if is_sync or self.world == 1:
            self.blk.step(x, step, is_sync)
        else:
            self.blk._check(self.dfp.LIB.dfp_step_patches(self.blk.h, ctypes.c_void_p(x.data_ptr()), int(step),
                                                          self.p0, self.p1))

    def stream_context(self):
        return torch.cuda.stream(self.blk.stream)

    def output(self):
        return self.blk.output()

    def close(self):
        self.blk.close()


def exchange(layers, transport, step, is_sync):
    """The exchange after `step` for the ranks in `layers` (the process's one rank with
    DistTransport; every emulated rank with LocalTransport, all on one stream), enqueued
    on the first layer's stream."""
    if layers[0].world == 1:
        return
    parity = step & 1
    cfg, world = layers[0].cfg, layers[0].world
    with layers[0].stream_context():
        if is_sync:
            for L in layers:
                halo_from_local(cfg, L.buffer, parity, L.rank, world)
            return
        pairs, fills = [], []
        for L in layers:
            pack, recv, fill = boundary_rows(cfg, L.buffer, parity, L.rank, world)
            pack()
            n = recv.numel() // world
            pairs.append(gathers(cfg, L.buffer, parity, L.rank, world) +
                         [(recv, recv[L.rank * n:(L.rank + 1) * n])])
            fills.append(fill)
        transport.all_gather(pairs)
        for fill in fills:
            fill()
