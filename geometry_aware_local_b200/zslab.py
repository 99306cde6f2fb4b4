"""One PACK3D volume split over several GPUs by z-slabs.

The operator of "Geometry Matters in Packed 3D Attention" shards along z:
with summary blocks one plane thick (b_z = 1) no block straddles two slabs,
a query's local window reaches only r_z planes past its slab (Key design 3),
and the compressed branch needs every summary of the volume (Key design 3:
every token attends to all M summaries).  Rank r of `world` owns the planes
[z0, z1) of the lattice and

1. sends the K_loc / V_loc rows of its first and last r_z planes to the ranks
   below and above and receives theirs (point-to-point: the halo);
2. runs the index map, summaries, RoPE and local attention on its slab
   extended by the received halo planes, as a lattice whose `origin` is the
   true z of its first plane, so every rotation uses true coordinates (Key
   design 1);
3. all-gathers the summaries of its own blocks; slabs are contiguous and in
   rank order, so the concatenation is the whole volume's summary array in
   its raster block order;
4. runs the query x summary stage with the gate for its own tokens against
   all M summaries (`pack3d_summary_attn_rows`).

A rank passes its own tokens (any packing; coordinates local to its slab, z
from 0) and gets their outputs in the same order.  The exchanges use
torch.distributed (NCCL between GPUs; any backend for the host logic).  This
module only moves and arranges tensors; every stage runs in the library's
kernels.  Halo tokens carry zero queries and gate logits (their outputs are
dropped) and zero compressed keys, values and scores (their summaries are
dropped).  `forward` composes the phases; `prepare`, `local_stage`,
`own_summaries`, `gather_summaries` and `global_stage` are the phases
themselves.
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
    extended lattice of Z_ext planes that starts at true plane z0 - lo."""
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


def take_slab(inp: Dict, p: SlabPlan):
    """Rank p.rank's tokens of a whole volume's inputs, in their input order, with z made local
    to the slab.  Returns (their indices in `inp`, their inputs)."""
    import torch
    z = inp["coords"][:, 0]
    idx = torch.nonzero((z >= p.z0) & (z < p.z1)).flatten()
    own = {k: inp[k].index_select(0, idx).contiguous() for k in NAMES}
    own["coords"][:, 0] -= p.z0
    return idx, own


def ext_config(cfg, p: SlabPlan):
    """Config of the extended lattice: Z_ext planes whose first one is true plane z0 - lo."""
    c = type(cfg).from_buffer_copy(cfg)
    c.Z = p.Z_ext
    c.origin[0] = cfg.origin[0] + p.z0 - p.lo
    return c


def boundary_rows(coords, p: SlabPlan):
    """Indices of this rank's tokens on its first r_z planes and on its last r_z planes, each in raster
    order over (z, y, x): what the ranks below and above receive as their halo."""
    import torch
    c = coords.long()
    order = torch.argsort((c[:, 0] * p.H + c[:, 1]) * p.W + c[:, 2])   # the slab's sites in raster order
    n = min(p.rz, p.planes) * p.plane_sites
    return order[:n], order[p.tokens - n:]


def exchange_halo(k_loc, v_loc, coords, p: SlabPlan, group=None):
    """Sends the K_loc / V_loc rows of this rank's first r_z planes to the rank below and of its last
    r_z planes to the rank above, and receives theirs.  Returns (below, above), tensors
    [lo * H * W, 2, Hkv, d_h] and [hi * H * W, 2, Hkv, d_h] (K then V) in raster order."""
    import torch
    import torch.distributed as dist
    first, last = boundary_rows(coords, p)
    kv = torch.stack([k_loc, v_loc], dim=1)
    below = kv.new_empty((p.lo * p.plane_sites,) + tuple(kv.shape[1:]))
    above = kv.new_empty((p.hi * p.plane_sites,) + tuple(kv.shape[1:]))
    ops = []
    if p.lo:
        ops.append(dist.P2POp(dist.isend, kv.index_select(0, first).contiguous(), p.rank - 1, group))
        ops.append(dist.P2POp(dist.irecv, below, p.rank - 1, group))
    if p.hi:
        ops.append(dist.P2POp(dist.isend, kv.index_select(0, last).contiguous(), p.rank + 1, group))
        ops.append(dist.P2POp(dist.irecv, above, p.rank + 1, group))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    return below, above


def prepare(inp: Dict, below, above, p: SlabPlan) -> Dict:
    """The extended lattice's inputs: this rank's tokens first (z shifted by lo), then the halo planes
    received from below (z = 0 .. lo-1) and from above (the last hi planes), each in raster order.
    Halo tokens get their K_loc / V_loc rows and zeros elsewhere."""
    import torch
    own = {k: inp[k] for k in NAMES}
    dev = own["q"].device
    n_lo, n_hi = p.lo * p.plane_sites, p.hi * p.plane_sites

    def plane_coords(z_from: int, count: int):
        idx = torch.arange(count, device=dev, dtype=torch.int64)
        return torch.stack([z_from + idx // p.plane_sites, (idx // p.W) % p.H, idx % p.W], dim=1).to(torch.int32)

    shift = torch.tensor([p.lo, 0, 0], dtype=torch.int32, device=dev)
    ext = {"coords": torch.cat([own["coords"] + shift, plane_coords(0, n_lo),
                                plane_coords(p.lo + p.planes, n_hi)])}

    def pad(t, halo_rows=None):
        zeros = t.new_zeros((n_lo + n_hi,) + tuple(t.shape[1:]))
        if halo_rows is not None:
            zeros = halo_rows
        return torch.cat([t, zeros])

    ext["k_loc"] = pad(own["k_loc"], torch.cat([below[:, 0], above[:, 0]]))
    ext["v_loc"] = pad(own["v_loc"], torch.cat([below[:, 1], above[:, 1]]))
    for k in ("q", "k_cmp", "v_cmp", "scores", "gate"):
        ext[k] = pad(own[k])
    return {k: v.contiguous() for k, v in ext.items()}


def own_summaries(k_sum, v_sum, p: SlabPlan, blocks_per_plane: int):
    """The summaries of this rank's own blocks (planes lo .. lo + planes - 1 of the extended lattice)."""
    a = p.lo * blocks_per_plane
    b = a + p.planes * blocks_per_plane
    return k_sum[a:b], v_sum[a:b]


def gather_summaries(k_own, v_own, p: SlabPlan, blocks_per_plane: int, group=None):
    """All ranks' own summaries, concatenated in rank order (= the volume's raster block order)."""
    import torch
    import torch.distributed as dist
    bounds = slab_bounds(p.Z, p.world)
    most = max(b - a for a, b in bounds) * blocks_per_plane
    kv = torch.stack([k_own, v_own], dim=1)
    padded = kv.new_zeros((most,) + tuple(kv.shape[1:]))
    padded[:kv.shape[0]] = kv
    parts = [torch.empty_like(padded) for _ in range(p.world)]
    dist.all_gather(parts, padded, group=group)
    allkv = torch.cat([parts[r][:(b - a) * blocks_per_plane] for r, (a, b) in enumerate(bounds)])
    return allkv[:, 0].contiguous(), allkv[:, 1].contiguous()


def local_stage(cfg_e, ext: Dict, err, stream=None):
    """Index map, summaries, RoPE and local attention on the extended lattice (library kernels).
    Returns q_rot, o_loc (every extended token) and k_sum, v_sum (every extended block)."""
    import torch

    from . import build_index, build_summaries, local_attn, rope_qk
    dev = ext["q"].device
    N, M, v = cfg_e.N, cfg_e.M, cfg_e.v
    g2p = torch.empty(N, dtype=torch.int32, device=dev)
    mem = torch.empty(M, v, dtype=torch.int32, device=dev)
    build_index(cfg_e, ext["coords"], g2p, mem, err, stream)
    k_sum = torch.empty(M, cfg_e.Hkv, cfg_e.d_h, dtype=ext["q"].dtype, device=dev)
    v_sum = torch.empty_like(k_sum)
    build_summaries(cfg_e, mem, ext["k_cmp"], ext["v_cmp"], ext["scores"], k_sum, v_sum, stream)
    q_rot, k_rot = torch.empty_like(ext["q"]), torch.empty_like(ext["k_loc"])
    rope_qk(cfg_e, ext["coords"], ext["q"], q_rot, ext["k_loc"], k_rot, stream)
    o_loc = torch.empty(N, cfg_e.Hq, cfg_e.d_h, dtype=torch.float32, device=dev)
    local_attn(cfg_e, g2p, q_rot, k_rot, ext["v_loc"], o_loc, err, stream)
    return q_rot, o_loc, k_sum, v_sum


def global_stage(cfg_e, tokens: int, q_rot, k_all, v_all, o_loc, gate, err, stream=None):
    """The query x summary stage and the gate for the first `tokens` extended rows (this rank's own)."""
    import torch

    from . import summary_attn_rows
    out = torch.empty_like(q_rot[:tokens])
    summary_attn_rows(cfg_e, tokens, k_all.shape[0], q_rot[:tokens], k_all, v_all, o_loc[:tokens],
                      gate[:tokens], out, err, stream)
    return out


def forward(cfg, inp: Dict, rank: int, world: int, group=None, stream=None):
    """This rank's part of the forward pass of the volume `cfg` split over `world` ranks: `inp` holds
    its own tokens (CUDA tensors, coordinates local to its slab); returns their outputs."""
    import torch

    from . import check_status
    p = make_plan(cfg, rank, world)
    if inp["q"].shape[0] != p.tokens:
        raise ValueError(f"rank {rank} owns {p.tokens} tokens, got {inp['q'].shape[0]}")
    cfg_e = ext_config(cfg, p)
    blocks_per_plane = (cfg.H // cfg.by) * (cfg.W // cfg.bx)
    err = torch.zeros(4, dtype=torch.int32, device=inp["q"].device)
    below, above = exchange_halo(inp["k_loc"], inp["v_loc"], inp["coords"], p, group)
    ext = prepare(inp, below, above, p)
    q_rot, o_loc, k_sum, v_sum = local_stage(cfg_e, ext, err, stream)
    k_own, v_own = own_summaries(k_sum, v_sum, p, blocks_per_plane)
    k_all, v_all = gather_summaries(k_own, v_own, p, blocks_per_plane, group)
    out = global_stage(cfg_e, p.tokens, q_rot, k_all, v_all, o_loc, ext["gate"], err, stream)
    st = check_status(err, stream)
    if st != 0:
        from . import Pack3DError
        raise Pack3DError(st, "z-slab forward")
    return out
