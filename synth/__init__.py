"""Seeded synthetic inputs for the PACK3D operator: lattices, packings and tensors.

This module is shared by the tests, the benchmark and the oracle checks. It holds
no arithmetic of the operator itself: it only decides *which* lattice site each
packed slot holds (the packing) and draws the per-site input values.

Workload recipe (the configurations of "Geometry Matters in Packed 3D Attention",
method section "Key design 1-3" and the scaling table, Table 4):

* Values are drawn per lattice site, in raster order over the lattice, from
  ``numpy.random.default_rng(seed)`` (PCG64), as float32 standard normals via
  ``Generator.standard_normal(dtype=float32)``.  Tensors are drawn in a fixed
  order: Q, K_loc, V_loc, K_cmp, V_cmp, block scores, gate logits.
* The output gradient dOut of the backward pass (the stress configuration's
  dOut ~ N(0,1)) is drawn the same way, per site in raster order, from its own
  generator ``default_rng(seed + 2)``, so the forward inputs do not change.
* Q/K/V draws are multiplied by ``value_scale`` (1 for the tiny case, 1/8 =
  1/sqrt(d_h) for the large volumes).  Scores and gate logits stay N(0,1).
* The per-site tensors are then permuted into packed order: packed slot ``p``
  holds lattice site ``site[p]``.  Every packing of one volume therefore carries
  the same physical field, which is what packing equivariance compares.
* bf16 tensors are the float32 draws rounded to nearest-even by torch; the
  oracle receives exactly those bf16 values, widened to float64.

Packings (the page lists raster, Morton/Z-order, block-contiguous and random):

* ``raster``  - site order ``(z*H + y)*W + x``.
* ``morton``  - sites sorted by a Morton key that interleaves coordinate bits from
  the least significant level up, x then y then z inside a level, skipping an
  axis once its bits are used up (a bijection for any lattice shape).
* ``block``   - blocks of ``bz x by x bx`` sites in raster order over the block
  grid, the sites of a block contiguous and raster-ordered inside it.
* ``random``  - ``default_rng(seed + 1).permutation(N)`` of the raster order.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

__all__ = [
    "Pack3DShape", "CONFIGS", "lattice_sites", "packing_sites", "coords_for",
    "draw_site_values", "make_inputs", "sample_rows", "make_dout",
]


@dataclasses.dataclass(frozen=True)
class Pack3DShape:
    """Shape and hyper-parameters of one operator instance."""
    Z: int
    H: int
    W: int
    Hq: int
    Hkv: int
    d_h: int = 64
    m_z: int = 11
    m_y: int = 11
    m_x: int = 10
    rope_base: float = 10000.0
    bz: int = 1
    by: int = 4
    bx: int = 4
    rz: int = 1
    ry: int = 3
    rx: int = 3
    dtype: str = "bf16"          # "f32" or "bf16"
    value_scale: float = 0.125   # multiplier on the Q/K/V draws
    packing: str = "raster"
    coord_scale: tuple = (1.0, 1.0, 1.0)   # per-axis RoPE coordinate scale (z, y, x)
    origin: tuple = (0, 0, 0)              # lattice origin in the rotation's frame (a sub-volume's offset)

    @property
    def N(self) -> int:
        return self.Z * self.H * self.W

    @property
    def v(self) -> int:
        return self.bz * self.by * self.bx

    @property
    def M(self) -> int:
        return self.N // self.v

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.d_h)

    def replace(self, **kw) -> "Pack3DShape":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny CPU-checkable case, three volumes (65k, 262k, 1M
# tokens) and the 65k repacking stress case.
CONFIGS: Dict[str, Pack3DShape] = {
    "tiny": Pack3DShape(Z=4, H=8, W=8, Hq=2, Hkv=1, rz=1, ry=1, rx=1,
                        dtype="f32", value_scale=1.0, packing="raster"),
    "65k": Pack3DShape(Z=16, H=64, W=64, Hq=8, Hkv=2, packing="morton"),
    "262k": Pack3DShape(Z=16, H=128, W=128, Hq=8, Hkv=2, packing="block"),
    "1m": Pack3DShape(Z=64, H=128, W=128, Hq=8, Hkv=2, packing="random"),
    "stress": Pack3DShape(Z=16, H=64, W=64, Hq=8, Hkv=2, packing="raster"),
    # The shape of the pages' Allen WTC-11 token grid (32 x 128 x 64), synthetic values.
    "allen": Pack3DShape(Z=32, H=128, W=64, Hq=8, Hkv=2, packing="block"),
    # Long query runs (4M and 8M tokens; inputs drawn on the device).
    "4m": Pack3DShape(Z=64, H=256, W=256, Hq=8, Hkv=2, packing="morton"),
    "8m": Pack3DShape(Z=128, H=256, W=256, Hq=8, Hkv=2, packing="morton"),
}
DEVICE_DRAWN = ("4m", "8m")

PACKINGS = ("raster", "morton", "block", "random", "block_morton")


def lattice_sites(Z: int, H: int, W: int) -> np.ndarray:
    """int32 [N,3] (z,y,x) of every lattice site in raster order."""
    z, y, x = np.meshgrid(np.arange(Z), np.arange(H), np.arange(W), indexing="ij")
    return np.stack([z.ravel(), y.ravel(), x.ravel()], axis=1).astype(np.int32)


def _morton_keys(Z: int, H: int, W: int, s: Optional[np.ndarray] = None) -> np.ndarray:
    """Morton code of each site (raster order by default) of a Z x H x W lattice."""
    if s is None:
        s = lattice_sites(Z, H, W)
    s = np.asarray(s).astype(np.int64)
    nbits = [max(1, (n - 1).bit_length()) for n in (Z, H, W)]
    key = np.zeros(s.shape[0], dtype=np.int64)
    out_bit = 0
    for level in range(max(nbits)):
        for axis in (2, 1, 0):          # x, then y, then z inside a level
            if level < nbits[axis]:
                key |= ((s[:, axis] >> level) & 1) << out_bit
                out_bit += 1
    return key


def packing_sites(Z: int, H: int, W: int, packing: str, seed: int = 0,
                  block=(1, 4, 4)) -> np.ndarray:
    """Raster site index held by each packed slot, int64 [N]."""
    N = Z * H * W
    if packing == "raster":
        return np.arange(N, dtype=np.int64)
    if packing == "morton":
        return np.argsort(_morton_keys(Z, H, W), kind="stable").astype(np.int64)
    if packing == "block":
        bz, by, bx = block
        if Z % bz or H % by or W % bx:
            raise ValueError("block packing needs block dims dividing the lattice")
        s = lattice_sites(Z, H, W).astype(np.int64)
        bid = ((s[:, 0] // bz) * (H // by) + s[:, 1] // by) * (W // bx) + s[:, 2] // bx
        inner = ((s[:, 0] % bz) * by + s[:, 1] % by) * bx + s[:, 2] % bx
        return np.argsort(bid * (bz * by * bx) + inner, kind="stable").astype(np.int64)
    if packing == "block_morton":
        # Two levels: blocks in Morton order over the block grid, sites in
        # Morton order inside each block.
        bz, by, bx = block
        if Z % bz or H % by or W % bx:
            raise ValueError("block_morton packing needs block dims dividing the lattice")
        s = lattice_sites(Z, H, W).astype(np.int64)
        outer = _morton_keys(Z // bz, H // by, W // bx, s // np.array([bz, by, bx]))
        # Morton rank (0 .. v-1) of each in-block offset, so blocks stay contiguous.
        rank = np.argsort(np.argsort(_morton_keys(bz, by, bx), kind="stable"), kind="stable")
        off = s % np.array([bz, by, bx])
        inner = rank[(off[:, 0] * by + off[:, 1]) * bx + off[:, 2]]
        return np.argsort(outer * (bz * by * bx) + inner, kind="stable").astype(np.int64)
    if packing == "random":
        return np.random.default_rng(seed + 1).permutation(N).astype(np.int64)
    raise ValueError(f"unknown packing {packing!r}")


def coords_for(shape: Pack3DShape, packing: Optional[str] = None, seed: int = 0) -> np.ndarray:
    """int32 [N,3] coordinates of the packed slots under ``packing``."""
    packing = packing or shape.packing
    sites = packing_sites(shape.Z, shape.H, shape.W, packing, seed,
                          (shape.bz, shape.by, shape.bx))
    return lattice_sites(shape.Z, shape.H, shape.W)[sites]


def draw_site_values(shape: Pack3DShape, seed: int = 0) -> Dict[str, np.ndarray]:
    """Per-lattice-site float32 draws in raster order (see module docstring)."""
    rng = np.random.default_rng(seed)
    N, Hq, Hkv, d = shape.N, shape.Hq, shape.Hkv, shape.d_h
    vs = np.float32(shape.value_scale)
    out = {}
    for name, heads in (("q", Hq), ("k_loc", Hkv), ("v_loc", Hkv),
                        ("k_cmp", Hkv), ("v_cmp", Hkv)):
        a = rng.standard_normal((N, heads, d), dtype=np.float32)
        if vs != 1:
            a *= vs
        out[name] = a
    out["scores"] = rng.standard_normal((N, Hkv), dtype=np.float32)
    out["gate"] = rng.standard_normal((N, Hq, 2), dtype=np.float32)
    return out


def make_inputs(shape: Pack3DShape, packing: Optional[str] = None, seed: int = 0,
                site_values: Optional[Dict[str, np.ndarray]] = None):
    """Packed torch CPU tensors for one operator call.

    Returns a dict with ``coords`` (int32 [N,3]) and ``q, k_loc, v_loc, k_cmp,
    v_cmp`` in ``shape.dtype`` plus float32 ``scores`` [N,Hkv] and ``gate``
    [N,Hq,2], all in packed order, and ``sites`` (int64 [N]).
    """
    import torch
    packing = packing or shape.packing
    sv = site_values if site_values is not None else draw_site_values(shape, seed)
    sites = packing_sites(shape.Z, shape.H, shape.W, packing, seed,
                          (shape.bz, shape.by, shape.bx))
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
    res = {"coords": torch.from_numpy(lattice_sites(shape.Z, shape.H, shape.W)[sites].copy()),
           "sites": torch.from_numpy(sites)}
    idx = torch.from_numpy(sites)
    for name in ("q", "k_loc", "v_loc", "k_cmp", "v_cmp"):
        res[name] = torch.from_numpy(sv[name]).index_select(0, idx).to(tdt).contiguous()
    for name in ("scores", "gate"):
        res[name] = torch.from_numpy(sv[name]).index_select(0, idx).contiguous()
    return res


def make_dout(shape: Pack3DShape, packing: Optional[str] = None, seed: int = 0, scale: float = 1.0):
    """Packed output gradient dOut [N, Hq, d_h] in ``shape.dtype`` (torch CPU tensor):
    ``scale`` times N(0,1) float32 draws per lattice site in raster order from
    ``default_rng(seed + 2)``, permuted like ``make_inputs``'s tensors."""
    import torch
    packing = packing or shape.packing
    rng = np.random.default_rng(seed + 2)
    a = rng.standard_normal((shape.N, shape.Hq, shape.d_h), dtype=np.float32)
    if scale != 1:
        a *= np.float32(scale)
    sites = packing_sites(shape.Z, shape.H, shape.W, packing, seed, (shape.bz, shape.by, shape.bx))
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
    return torch.from_numpy(a).index_select(0, torch.from_numpy(sites)).to(tdt).contiguous()


def make_inputs_on_device(shape: Pack3DShape, packing: Optional[str] = None, seed: int = 0,
                          device="cuda"):
    """The same inputs as ``make_inputs`` in kind and distribution, drawn on the device.

    For volumes whose float32 host draws would not fit the host (4M and 8M
    tokens): the coordinates of ``packing`` come from the host as above, the
    values are drawn in packed order by a seeded torch generator on ``device``
    (N(0,1) times ``value_scale`` for Q/K/V, N(0,1) for scores and gate).  The
    values differ from ``make_inputs``'s; no parity check uses these volumes."""
    import torch
    packing = packing or shape.packing
    sites = packing_sites(shape.Z, shape.H, shape.W, packing, seed, (shape.bz, shape.by, shape.bx))
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
    gen = torch.Generator(device=device).manual_seed(seed)
    N, Hq, Hkv, d = shape.N, shape.Hq, shape.Hkv, shape.d_h
    res = {"coords": torch.from_numpy(lattice_sites(shape.Z, shape.H, shape.W)[sites].copy()).to(device)}
    for name, heads in (("q", Hq), ("k_loc", Hkv), ("v_loc", Hkv), ("k_cmp", Hkv), ("v_cmp", Hkv)):
        x = torch.randn((N, heads, d), generator=gen, device=device, dtype=torch.float32)
        if shape.value_scale != 1:
            x *= shape.value_scale
        res[name] = x.to(tdt)
        del x
    res["scores"] = torch.randn((N, Hkv), generator=gen, device=device, dtype=torch.float32)
    res["gate"] = torch.randn((N, Hq, 2), generator=gen, device=device, dtype=torch.float32)
    return res


def sample_rows(N: int, count: int, seed: int = 0) -> np.ndarray:
    """Sorted seeded sample of packed row indices, always including 0 and N-1."""
    if count >= N:
        return np.arange(N, dtype=np.int64)
    rng = np.random.default_rng(seed + 7)
    rows = rng.choice(N, size=count, replace=False)
    rows[0], rows[1] = 0, N - 1
    return np.unique(rows).astype(np.int64)
