"""One PACK3D volume split over several GPUs by z-slabs.

The operator of "Geometry Matters in Packed 3D Attention" shards along z:
with summary blocks one plane thick (b_z = 1) no block straddles two slabs,
a query's local window reaches only r_z planes past its slab (Key design 3),
and the compressed branch needs every summary of the volume (Key design 3:
every token attends to all M summaries).  Rank r of `world` owns the planes
[z0, z1) of the lattice and runs, per step:

1. the local keys and values of its first and last r_z planes, gathered in
   raster order through its index map (`pack3d_gather_rows`), go to the ranks
   below and above, and theirs arrive straight into its halo rows (NCCL
   point-to-point);
2. summaries, RoPE and local attention run on its slab extended by the halo
   planes, a lattice whose config `origin` is the true z of its first plane,
   so every rotation uses true coordinates (Key design 1);
3. the summaries of its own blocks (one contiguous range: blocks are planes of
   b_z = 1) are all-gathered; slabs are contiguous and in rank order, so the
   result is the whole volume's summary array in raster block order;
4. the query x summary stage and the gate run for its own tokens against all
   M summaries (`pack3d_summary_attn_rows`).

`Plan` sets a rank up once for its fixed coordinates: the extended lattice's
coordinates and index map (built once; the geometry does not change between
steps), and every buffer.  The caller writes its own tokens' inputs into
`Plan.inputs()` (views of the extended arrays, any order within the slab) and
calls `Plan.forward()`.  Halo tokens carry zero queries, gate logits,
compressed keys, values and scores; their outputs and summaries are dropped.
Every per-step data movement is a library kernel or a NCCL call; PyTorch only
holds the buffers and runs the collectives.  The phases are also callable one
by one (`pack_halo`, `halo_views`, `local`, `summary_part`, `attend`), which
is how a single process can run every rank's work in turn.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Tuple

NAMES = ("coords", "q", "k_loc", "v_loc", "k_cmp", "v_cmp", "scores", "gate")


def slab_bounds(Z: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous z ranges [z0, z1) of the ranks, in rank order, sizes differing by at most one plane."""
    if world < 1 or Z < world:
        raise ValueError(f"cannot split {Z} planes over {world} ranks")
    base, extra = divmod(Z, world)
    out, z = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((z, z + n))
        z += n
    return out


@dataclasses.dataclass(frozen=True)
class SlabPlan:
    """Rank `rank`'s part of a Z x H x W volume: its planes [z0, z1), the halo
    planes it receives from below (`lo`) and from above (`hi`), and the
    extended lattice of Z_ext planes that starts at true plane z0 - lo.  Rows of
    the extended arrays: the rank's own tokens first, then the `lo` planes below
    and the `hi` planes above, each in raster order."""
    Z: int
    H: int
    W: int
    rz: int
    rank: int
    world: int
    z0: int
    z1: int
    lo: int
    hi: int

    @property
    def planes(self) -> int:
        return self.z1 - self.z0

    @property
    def Z_ext(self) -> int:
        return self.planes + self.lo + self.hi

    @property
    def plane_sites(self) -> int:
        return self.H * self.W

    @property
    def tokens(self) -> int:
        return self.planes * self.plane_sites

    @property
    def halo_below(self) -> Tuple[int, int]:
        """Rows of the extended arrays that hold the planes received from below."""
        return self.tokens, self.tokens + self.lo * self.plane_sites

    @property
    def halo_above(self) -> Tuple[int, int]:
        """Rows of the extended arrays that hold the planes received from above."""
        a = self.tokens + self.lo * self.plane_sites
        return a, a + self.hi * self.plane_sites

    @property
    def send_below(self) -> Tuple[int, int]:
        """Sites (raster over the extended lattice) of the own planes the rank below receives."""
        a = self.lo * self.plane_sites
        return a, a + min(self.rz, self.planes) * self.plane_sites

    @property
    def send_above(self) -> Tuple[int, int]:
        """Sites (raster over the extended lattice) of the own planes the rank above receives."""
        b = (self.lo + self.planes) * self.plane_sites
        return b - min(self.rz, self.planes) * self.plane_sites, b

    def own_blocks(self, blocks_per_plane: int) -> Tuple[int, int]:
        """The extended lattice's blocks that are the rank's own (raster block order)."""
        return self.lo * blocks_per_plane, (self.lo + self.planes) * blocks_per_plane


def make_plan(cfg, rank: int, world: int) -> SlabPlan:
    """Rank `rank`'s slab of the volume `cfg` describes (whose origin the slabs inherit)."""
    Z, H, W, rz = cfg.Z, cfg.H, cfg.W, cfg.rz
    if cfg.bz != 1:
        raise ValueError("the z-slab split needs summary blocks one plane thick (bz = 1)")
    bounds = slab_bounds(Z, world)
    if world > 1 and min(b - a for a, b in bounds) < rz:
        raise ValueError(f"every slab needs at least rz = {rz} planes (the halo comes from the neighbours only)")
    z0, z1 = bounds[rank]
    return SlabPlan(Z, H, W, rz, rank, world, z0, z1, min(rz, z0), min(rz, Z - z1))


def ext_config(cfg, p: SlabPlan):
    """Config of the extended lattice: Z_ext planes whose first one is true plane z0 - lo."""
    c = type(cfg).from_buffer_copy(cfg)
    c.Z = p.Z_ext
    c.origin[0] = cfg.origin[0] + p.z0 - p.lo
    return c


def ext_coords(coords, p: SlabPlan):
    """Coordinates of the extended lattice's rows: the own tokens' (z local to the slab, shifted
    by lo), then the halo planes below and above in raster order."""
    import torch
    dev = coords.device

    def plane_coords(z_from: int, count: int):
        idx = torch.arange(count, device=dev, dtype=torch.int64)
        return torch.stack([z_from + idx // p.plane_sites, (idx // p.W) % p.H, idx % p.W], dim=1).to(torch.int32)

    shift = torch.tensor([p.lo, 0, 0], dtype=torch.int32, device=dev)
    return torch.cat([coords.to(torch.int32) + shift, plane_coords(0, p.lo * p.plane_sites),
                      plane_coords(p.lo + p.planes, p.hi * p.plane_sites)]).contiguous()


def summary_parts(cfg, world: int) -> List[Tuple[int, int, int]]:
    """How the ranks' summaries are all-gathered: a part of `most` summaries per rank (the
    largest rank's count), taken from its extended summary array at `start`, whose own blocks
    begin `offset` summaries into it.  Returns [(start, offset, count)] in rank order; with
    even slabs every offset is 0 and every count equals most.  A smaller rank's part extends
    into its halo blocks (above it, or below it for the last rank), which are dropped."""
    bpp = (cfg.H // cfg.by) * (cfg.W // cfg.bx)
    plans = [make_plan(cfg, r, world) for r in range(world)]
    most = max(p.planes for p in plans) * bpp
    out = []
    for p in plans:
        a, b = p.own_blocks(bpp)
        start = a if a + most <= p.Z_ext * bpp else b - most
        out.append((start, a - start, b - a))
    return out


def take_slab(inp: Dict, p: SlabPlan):
    """Rank p.rank's tokens of a whole volume's inputs, in their input order, with z made local
    to the slab.  Returns (their indices in `inp`, their inputs).  (For tests and examples that
    hold a whole volume in one process.)"""
    import torch
    z = inp["coords"][:, 0]
    idx = torch.nonzero((z >= p.z0) & (z < p.z1)).flatten()
    own = {k: inp[k].index_select(0, idx).contiguous() for k in NAMES}
    own["coords"][:, 0] -= p.z0
    return idx, own


class Plan:
    """One rank's z-slab forward, set up once for the rank's fixed token coordinates.

    `coords` (int32 [tokens, 3], on the rank's CUDA device) are the rank's own
    tokens' lattice coordinates with z local to its slab (0 .. planes-1); their
    order is the order of `inputs()` and of the output.  With world > 1 the
    exchanges run on `group` (torch.distributed, NCCL between GPUs); a one-rank
    plan needs no process group.  `stream` (None: torch's current stream; a
    torch.cuda.Stream or a raw cudaStream_t) carries every phase and, through
    torch's current-stream context, the exchanges; with an explicit stream the
    caller orders its writes of `inputs()` before `forward` on that stream."""

    def __init__(self, cfg, coords, rank: int, world: int, group=None, stream=None):
        import torch

        from . import BF16, Pack3DError, build_index, check_status, validate
        st = validate(cfg)
        if st != 0:
            raise Pack3DError(st, "z-slab config")
        self.cfg, self.group, self.stream = cfg, group, stream
        self.p = p = make_plan(cfg, rank, world)
        if coords.shape[0] != p.tokens:
            raise ValueError(f"rank {rank} owns {p.tokens} tokens, got {coords.shape[0]}")
        self.cfg_e = ce = ext_config(cfg, p)
        dev = coords.device
        dt = torch.bfloat16 if cfg.dtype == BF16 else torch.float32
        N, M, Hq, Hkv, d = ce.N, ce.M, cfg.Hq, cfg.Hkv, cfg.d_h

        def zeros(*shape, dtype=dt):
            return torch.zeros(shape, dtype=dtype, device=dev)

        # Extended inputs; the halo rows stay zero except K_loc / V_loc, received every step.
        self.ext = {"coords": ext_coords(coords, p), "q": zeros(N, Hq, d), "k_loc": zeros(N, Hkv, d),
                    "v_loc": zeros(N, Hkv, d), "k_cmp": zeros(N, Hkv, d), "v_cmp": zeros(N, Hkv, d),
                    "scores": zeros(N, Hkv, dtype=torch.float32), "gate": zeros(N, Hq, 2, dtype=torch.float32)}
        self.err = torch.zeros(4, dtype=torch.int32, device=dev)
        self.g2p = torch.empty(N, dtype=torch.int32, device=dev)
        self.members = torch.empty(M, ce.v, dtype=torch.int32, device=dev)
        build_index(ce, self.ext["coords"], self.g2p, self.members, self.err, stream)
        st = check_status(self.err, stream)
        if st != 0:
            raise Pack3DError(st, "z-slab index map (the coordinates must cover the slab once each)")
        self.q_rot, self.k_rot = torch.empty_like(self.ext["q"]), torch.empty_like(self.ext["k_loc"])
        self.o_loc = zeros(N, Hq, d, dtype=torch.float32)
        self.k_sum, self.v_sum = zeros(M, Hkv, d), zeros(M, Hkv, d)
        self.out = zeros(p.tokens, Hq, d)
        # Halo send buffers and the rows of the extended arrays they are gathered from (a slice
        # of the index map: the boundary planes' sites in raster order).
        self.send = {}
        for side, (a, b), n in (("below", p.send_below, p.lo), ("above", p.send_above, p.hi)):
            if n:
                self.send[side] = (self.g2p[a:b], zeros(b - a, Hkv, d), zeros(b - a, Hkv, d))
        # The whole volume's summaries: gathered straight into k_all / v_all with even slabs, else
        # into padded parts and compacted by a row gather.
        parts = summary_parts(cfg, world)
        self.part = parts[rank]
        self.most = max(c for _, _, c in parts)
        M_all = sum(c for _, _, c in parts)
        if world == 1:   # the rank's own summaries are the volume's: no gather, no copy
            self.k_all, self.v_all = self.k_sum, self.v_sum
        else:
            self.k_all, self.v_all = zeros(M_all, Hkv, d), zeros(M_all, Hkv, d)
        self.uneven = any(o != 0 or c != self.most for _, o, c in parts)
        if self.uneven:
            self.k_pad, self.v_pad = zeros(self.most * world, Hkv, d), zeros(self.most * world, Hkv, d)
            self.compact = torch.cat([torch.arange(r * self.most + o, r * self.most + o + c, dtype=torch.int32)
                                      for r, (_, o, c) in enumerate(parts)]).to(dev)
        # The buffers above were filled on torch's current stream; the phases run on `stream`.
        if stream is not None:
            torch.cuda.synchronize(dev)

    def _on_stream(self):
        """Context in which torch.distributed calls order themselves after the phases' kernels:
        NCCL waits for torch's current stream, so that must be the plan's stream."""
        import contextlib

        import torch
        if self.stream is None:
            return contextlib.nullcontext()
        s = self.stream
        return torch.cuda.stream(torch.cuda.ExternalStream(s) if isinstance(s, int) else s)

    def inputs(self) -> Dict:
        """Views of the extended arrays' own rows, to be written before `forward` (in the order
        of the coordinates the plan was made with)."""
        t = self.p.tokens
        return {k: v[:t] for k, v in self.ext.items() if k != "coords"}

    # ---- the phases ----------------------------------------------------------------------------
    def pack_halo(self):
        """Gathers the boundary planes' K_loc / V_loc rows into the send buffers (raster order)."""
        from . import gather_rows
        for idx, ks, vs in self.send.values():
            gather_rows(idx, self.ext["k_loc"], ks, self.stream)
            gather_rows(idx, self.ext["v_loc"], vs, self.stream)

    def halo_views(self):
        """(below, above): None, or the (K_loc, V_loc) row views the neighbour's planes go to."""
        out = []
        for a, b in (self.p.halo_below, self.p.halo_above):
            out.append((self.ext["k_loc"][a:b], self.ext["v_loc"][a:b]) if b > a else None)
        return tuple(out)

    def local(self):
        """Summaries, RoPE and local attention on the extended lattice."""
        from . import build_summaries, local_attn, rope_qk
        e, ce = self.ext, self.cfg_e
        build_summaries(ce, self.members, e["k_cmp"], e["v_cmp"], e["scores"], self.k_sum, self.v_sum, self.stream)
        rope_qk(ce, e["coords"], e["q"], self.q_rot, e["k_loc"], self.k_rot, self.stream)
        local_attn(ce, self.g2p, self.q_rot, self.k_rot, e["v_loc"], self.o_loc, self.err, self.stream)

    def summary_part(self):
        """The rows of k_sum / v_sum this rank contributes to the all-gather (its own blocks, plus
        halo blocks up to the common part size when slabs are uneven)."""
        start = self.part[0]
        return self.k_sum[start:start + self.most], self.v_sum[start:start + self.most]

    def attend(self):
        """The query x summary stage and the gate for the own tokens against k_all / v_all."""
        from . import summary_attn_rows
        t = self.p.tokens
        summary_attn_rows(self.cfg_e, t, self.k_all.shape[0], self.q_rot[:t], self.k_all, self.v_all,
                          self.o_loc[:t], self.ext["gate"][:t], self.out, self.err, self.stream)
        return self.out

    # ---- the exchanges (NCCL between GPUs) ------------------------------------------------------
    def exchange_halo(self):
        if self.p.world == 1:
            return
        import torch.distributed as dist
        p, ops = self.p, []
        below, above = self.halo_views()
        for side, peer, recv in (("below", p.rank - 1, below), ("above", p.rank + 1, above)):
            if side in self.send:
                _, ks, vs = self.send[side]
                ops += [dist.P2POp(dist.isend, ks, peer, self.group), dist.P2POp(dist.isend, vs, peer, self.group),
                        dist.P2POp(dist.irecv, recv[0], peer, self.group),
                        dist.P2POp(dist.irecv, recv[1], peer, self.group)]
        if ops:
            with self._on_stream():
                for req in dist.batch_isend_irecv(ops):
                    req.wait()

    def gather_summaries(self):
        import torch.distributed as dist

        from . import gather_rows
        if self.p.world == 1:
            return
        k_part, v_part = self.summary_part()
        with self._on_stream():
            if not self.uneven:
                dist.all_gather_into_tensor(self.k_all, k_part, group=self.group)
                dist.all_gather_into_tensor(self.v_all, v_part, group=self.group)
                return
            dist.all_gather_into_tensor(self.k_pad, k_part, group=self.group)
            dist.all_gather_into_tensor(self.v_pad, v_part, group=self.group)
        gather_rows(self.compact, self.k_pad, self.k_all, self.stream)
        gather_rows(self.compact, self.v_pad, self.v_all, self.stream)

    def forward(self):
        """One step of the rank's forward pass; returns its tokens' outputs [tokens, Hq, d_h]."""
        from . import Pack3DError, check_status
        self.pack_halo()
        self.exchange_halo()
        self.local()
        self.gather_summaries()
        out = self.attend()
        st = check_status(self.err, self.stream)
        if st != 0:
            raise Pack3DError(st, "z-slab forward")
        return out


def forward(cfg, inp: Dict, rank: int, world: int, group=None, stream=None):
    """One rank's forward pass of the volume `cfg` split over `world` ranks, set up for this call
    only: `inp` holds its own tokens (CUDA tensors, coordinates local to its slab)."""
    plan = Plan(cfg, inp["coords"], rank, world, group, stream)
    for k, v in plan.inputs().items():
        v.copy_(inp[k])
    return plan.forward()
