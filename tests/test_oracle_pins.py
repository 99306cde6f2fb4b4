"""Pins of the float64 oracle against facts the pages and mathematics fix.

Each test checks the oracle against something other than itself: an identity
stated on the pages ("Geometry Matters in Packed 3D Attention": the relative-
position identity and Proposition 1 of Key design 1, Proposition 2 of Key
design 2), a closed form, a special case that reduces to a library routine
(torch's float64 scaled-dot-product attention, scipy's softmax, numpy complex
exponentials), or brute force on a tiny lattice.
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth

TINY = synth.CONFIGS["tiny"]


def small(**kw):
    base = dict(Z=3, H=8, W=8, Hq=4, Hkv=2, rz=1, ry=2, rx=2, dtype="f32", value_scale=1.0)
    base.update(kw)
    return synth.Pack3DShape(**base)


def rope_complex(s, coords, x):
    """Axial RoPE as complex multiplication of pair (x0 + i x1) by exp(i theta).

    RoFormer's complex form of a 2x2 rotation, with the per-axis frequency
    reading base^(-r/m_a) and pairs ordered z, y, x.
    """
    x = np.asarray(x, np.float64)
    n, h, d = x.shape
    z = x[..., 0::2] + 1j * x[..., 1::2]
    theta = np.zeros((n, d // 2))
    p0 = 0
    for axis, m in enumerate((s.m_z, s.m_y, s.m_x)):
        freqs = s.rope_base ** (-np.arange(m) / m)
        theta[:, p0:p0 + m] = np.asarray(coords, np.float64)[:, axis:axis + 1] * freqs[None, :]
        p0 += m
    z = z * np.exp(1j * theta)[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def rope_matrix(s, c):
    """R(c) as a d_h x d_h matrix, assembled by rotating the unit vectors."""
    d = s.d_h
    eye = np.eye(d).reshape(d, 1, d)
    coords = np.tile(np.asarray(c, np.int32), (d, 1))
    return oracle.rotate(s, coords, eye).reshape(d, d).T


def sdpa64(q, k, v, scale, mask=None):
    """torch float64 scaled-dot-product attention; q [n,h,d], k/v [m,h,d]."""
    qt = torch.from_numpy(np.ascontiguousarray(q)).permute(1, 0, 2)
    kt = torch.from_numpy(np.ascontiguousarray(k)).permute(1, 0, 2)
    vt = torch.from_numpy(np.ascontiguousarray(v)).permute(1, 0, 2)
    m = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
    return o.permute(1, 0, 2).numpy()


def expand_kv(s, kv):
    """Repeat kv heads so q head h reads kv head floor(h*Hkv/Hq)."""
    idx = [(h * s.Hkv) // s.Hq for h in range(s.Hq)]
    return np.asarray(kv)[:, idx, :]


# ---------------------------------------------------------------- RoPE -----

def test_rope_orthogonal_and_identity_at_origin():
    rng = np.random.default_rng(1)
    assert np.abs(rope_matrix(TINY, (0, 0, 0)) - np.eye(64)).max() == 0.0
    for _ in range(20):
        c = rng.integers(-300, 300, size=3)
        R = rope_matrix(TINY, c)
        assert np.abs(R.T @ R - np.eye(64)).max() < 1e-13


def test_rope_relative_position_identity():
    # R(c_i)^T R(c_j) = R(c_j - c_i) (Key design 1).
    rng = np.random.default_rng(2)
    for _ in range(30):
        ci, cj = rng.integers(0, 200, size=3), rng.integers(0, 200, size=3)
        lhs = rope_matrix(TINY, ci).T @ rope_matrix(TINY, cj)
        rhs = rope_matrix(TINY, cj - ci)
        assert np.abs(lhs - rhs).max() < 1e-12


def test_rope_axis_blocks():
    # Direct sum over z, y, x with m = (11, 11, 10) planes (Key design 1).
    s = TINY
    bounds = [(0, 22), (22, 44), (44, 64)]
    for axis in range(3):
        c = [0, 0, 0]
        c[axis] = 5
        R = rope_matrix(s, c)
        lo, hi = bounds[axis]
        off = R.copy()
        off[lo:hi, lo:hi] = 0
        assert np.abs(off - np.eye(64) * (1 - np.isin(np.arange(64), np.arange(lo, hi)))).max() == 0
        blk = R[lo:hi, lo:hi]
        # 2x2 rotations on adjacent pairs; none is the identity for a nonzero coordinate.
        for p in range(0, hi - lo, 2):
            b = blk[p:p + 2, p:p + 2]
            assert abs(b[0, 0] - b[1, 1]) < 1e-15 and abs(b[0, 1] + b[1, 0]) < 1e-15
            assert abs(b[0, 0] ** 2 + b[1, 0] ** 2 - 1) < 1e-14


def test_rope_untouched_remainder_dims():
    s = TINY.replace(m_z=8, m_y=8, m_x=8)   # 48 rotated dims, 16 left alone
    R = rope_matrix(s, (7, 3, 9))
    assert np.abs(R[48:, :] - np.eye(64)[48:, :]).max() == 0
    assert np.abs(R[:, 48:] - np.eye(64)[:, 48:]).max() == 0


def test_rope_matches_complex_form():
    rng = np.random.default_rng(3)
    coords = rng.integers(0, 128, size=(50, 3)).astype(np.int32)
    x = rng.standard_normal((50, 3, 64))
    assert np.abs(oracle.rotate(TINY, coords, x) - rope_complex(TINY, coords, x)).max() < 1e-12


@pytest.mark.parametrize("scale,m", [((1 / 31, 1 / 127, 1 / 63), (11, 11, 10)),   # normalised coordinates
                                     ((2.5, 1.0, 1.0), (11, 11, 10)),             # z rescaled
                                     ((1.0, 1.0, 1.0), (6, 13, 13)),              # z-light allocation
                                     ((1.0, 1.0, 1.0), (16, 8, 8))])              # z-heavy allocation
def test_rope_coordinate_scale_and_allocation_match_complex_form(scale, m):
    # A coordinate scale is the same rotation at the scaled (fractional) coordinate.
    s = TINY.replace(Z=32, H=128, W=64, m_z=m[0], m_y=m[1], m_x=m[2], coord_scale=scale)
    rng = np.random.default_rng(5)
    coords = np.stack([rng.integers(0, n, 40) for n in (s.Z, s.H, s.W)], axis=1).astype(np.int32)
    x = rng.standard_normal((40, 2, 64))
    expect = rope_complex(s, coords.astype(np.float64) * np.asarray(scale), x)
    assert np.abs(oracle.rotate(s, coords, x) - expect).max() < 1e-12


@pytest.mark.parametrize("origin", [(7, 0, 0), (3, -5, 11)])
def test_rope_origin_is_rotation_at_true_coordinate(origin):
    # A lattice that is one part of a larger volume (a z-slab) rotates its local site c by
    # R(origin + c): the rotation is driven by true coordinates (Key design 1).
    s = TINY.replace(origin=origin)
    rng = np.random.default_rng(9)
    coords = np.stack([rng.integers(0, n, 40) for n in (s.Z, s.H, s.W)], axis=1).astype(np.int32)
    x = rng.standard_normal((40, 2, 64))
    expect = rope_complex(s, coords + np.asarray(origin), x)
    assert np.abs(oracle.rotate(s, coords, x) - expect).max() < 1e-12
    assert np.abs(oracle.rotate(s, coords, x) - oracle.rotate(TINY, coords, x)).max() > 1e-3


# ------------------------------------------------------------ index map -----

@pytest.mark.parametrize("packing", synth.PACKINGS)
def test_index_map_brute_force(packing):
    s = small()
    coords = synth.coords_for(s, packing)
    st, g2p, mem = oracle.build_index(s, coords)
    assert st == 0
    for i, (z, y, x) in enumerate(coords):
        assert g2p[(z * s.H + y) * s.W + x] == i
    nby, nbx = s.H // s.by, s.W // s.bx
    for j in range(s.M):
        jz, jy, jx = j // (nby * nbx), (j // nbx) % nby, j % nbx
        t = 0
        for tz, ty, tx in itertools.product(range(s.bz), range(s.by), range(s.bx)):
            site = ((jz * s.bz + tz), (jy * s.by + ty), (jx * s.bx + tx))
            assert tuple(coords[mem[j, t]]) == site
            t += 1


def test_index_map_closed_forms():
    s = small()
    st, g2p, mem = oracle.build_index(s, synth.coords_for(s, "raster"))
    assert st == 0 and np.array_equal(g2p, np.arange(s.N))
    st, g2p, mem = oracle.build_index(s, synth.coords_for(s, "block"))
    assert st == 0 and np.array_equal(mem.ravel(), np.arange(s.N))


def test_index_map_rejects_bad_coords():
    s = small()
    c = synth.coords_for(s, "random").copy()
    c[5] = c[9]
    assert oracle.build_index(s, c)[0] == 2
    c = synth.coords_for(s, "raster").copy()
    c[3, 1] = s.H
    assert oracle.build_index(s, c)[0] == 1
    c[3, 1] = -1
    assert oracle.build_index(s, c)[0] == 1


def test_packings_are_bijections_with_expected_locality():
    s = synth.CONFIGS["65k"]
    for p in synth.PACKINGS:
        sites = synth.packing_sites(s.Z, s.H, s.W, p)
        assert np.array_equal(np.sort(sites), np.arange(s.N))
    # Morton: the first 8 slots form the 2x2x2 cube at the origin.
    c = synth.coords_for(s, "morton")
    assert sorted(map(tuple, c[:8])) == sorted(itertools.product(range(2), range(2), range(2)))
    # Two-level block Morton: every run of v slots is one block, walked in Morton order
    # inside it; the first four blocks are the 2x2 block square at the origin.
    c = synth.coords_for(s, "block_morton")
    blocks = c // np.array([s.bz, s.by, s.bx])
    for k in range(0, s.N, s.v):
        assert (blocks[k:k + s.v] == blocks[k]).all()
    assert sorted(map(tuple, blocks[0:4 * s.v:s.v])) == [(0, 0, 0), (0, 0, 1), (0, 1, 0), (0, 1, 1)]
    assert [tuple(x) for x in c[:4]] == [(0, 0, 0), (0, 0, 1), (0, 1, 0), (0, 1, 1)]


# -------------------------------------------------------------- summaries ---

def _summary_case(s, packing="random", seed=0):
    inp = synth.make_inputs(s, packing, seed)
    st, g2p, mem = oracle.build_index(s, inp["coords"])
    assert st == 0
    return inp, g2p, mem


def test_proposition_2_identity():
    # (q_i^R)^T k~_j = sum_u a_ju q_i^T R(c_u - c_i) k_u  (Key design 2).
    s = small()
    inp, g2p, mem = _summary_case(s)
    coords = inp["coords"].numpy()
    ks, vs = oracle.summaries(s, coords, mem, inp["k_cmp"], inp["v_cmp"], inp["scores"])
    kc = oracle.as_f64(inp["k_cmp"])
    sc = oracle.as_f64(inp["scores"])
    rng = np.random.default_rng(4)
    for _ in range(10):
        i = int(rng.integers(s.N))
        j = int(rng.integers(s.M))
        g = int(rng.integers(s.Hkv))
        q = rng.standard_normal((1, 1, 64))
        qr = oracle.rotate(s, coords[i:i + 1], q)[0, 0]
        lhs = qr @ ks[j, g]
        a = scipy.special.softmax(sc[mem[j], g])
        disp = (coords[mem[j]] - coords[i]).astype(np.int32)
        rk = oracle.rotate(s, disp, kc[mem[j], g][:, None, :])[:, 0, :]
        rhs = float(np.sum(a * (rk @ q[0, 0])))
        assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(rhs))


def test_summaries_weights_are_block_softmax():
    s = small()
    inp, g2p, mem = _summary_case(s)
    coords = inp["coords"].numpy()
    ks, vs = oracle.summaries(s, coords, mem, inp["k_cmp"], inp["v_cmp"], inp["scores"])
    vc, sc = oracle.as_f64(inp["v_cmp"]), oracle.as_f64(inp["scores"])
    kr = rope_complex(s, coords, oracle.as_f64(inp["k_cmp"]))
    for j in range(s.M):
        for g in range(s.Hkv):
            a = scipy.special.softmax(sc[mem[j], g])
            assert np.abs(vs[j, g] - a @ vc[mem[j], g]).max() < 1e-13
            assert np.abs(ks[j, g] - a @ kr[mem[j], g]).max() < 1e-12


def test_summaries_uniform_scores_mean_pool_and_unit_blocks():
    s = small()
    inp, g2p, mem = _summary_case(s)
    coords = inp["coords"].numpy()
    zero = np.zeros((s.N, s.Hkv))
    ks, vs = oracle.summaries(s, coords, mem, inp["k_cmp"], inp["v_cmp"], zero)
    vc = oracle.as_f64(inp["v_cmp"])
    assert np.abs(vs - vc[mem].mean(axis=1)).max() < 1e-14
    s1 = s.replace(by=1, bx=1)
    st, g2p1, mem1 = oracle.build_index(s1, coords)
    ks1, vs1 = oracle.summaries(s1, coords, mem1, inp["k_cmp"], inp["v_cmp"], inp["scores"])
    order = mem1[:, 0]
    assert np.abs(vs1[:, :, :] - vc[order]).max() == 0
    assert np.abs(ks1 - rope_complex(s, coords, oracle.as_f64(inp["k_cmp"]))[order]).max() < 1e-12


# ------------------------------------------------- summary-centre variant -----
# The cheaper variant the summary page names (contribution 2, "Future
# Directions" 3): pooled key unrotated, then rotated by the block centre.

def _block_centres(s):
    """Geometric centre of every block (raster over the block grid), fractional."""
    nbz, nby, nbx = s.Z // s.bz, s.H // s.by, s.W // s.bx
    jz, jy, jx = np.meshgrid(np.arange(nbz), np.arange(nby), np.arange(nbx), indexing="ij")
    return np.stack([jz.ravel() * s.bz + (s.bz - 1) / 2, jy.ravel() * s.by + (s.by - 1) / 2,
                     jx.ravel() * s.bx + (s.bx - 1) / 2], axis=1)


def test_summary_center_unit_blocks_equal_token_before():
    s = small(by=1, bx=1)
    inp, g2p, mem = _summary_case(s)
    coords = inp["coords"].numpy()
    kt, vt = oracle.summaries(s, coords, mem, inp["k_cmp"], inp["v_cmp"], inp["scores"])
    kc, vc = oracle.summaries(s, coords, mem, inp["k_cmp"], inp["v_cmp"], inp["scores"], center=True)
    assert np.abs(kc - kt).max() < 1e-12 and np.abs(vc - vt).max() == 0


@pytest.mark.parametrize("blocks", [(1, 4, 4), (2, 2, 2), (1, 2, 4)])
def test_summary_center_is_pooled_key_rotated_at_block_centre(blocks):
    s = small(Z=4, bz=blocks[0], by=blocks[1], bx=blocks[2])
    inp, g2p, mem = _summary_case(s, seed=7)
    coords = inp["coords"].numpy()
    kc = oracle.as_f64(inp["k_cmp"])
    a = scipy.special.softmax(oracle.as_f64(inp["scores"])[mem], axis=1)      # [M, v, Hkv]
    pooled = np.einsum("jug,jugd->jgd", a, kc[mem])
    expect = rope_complex(s, _block_centres(s), pooled)
    got, _ = oracle.summaries(s, coords, mem, inp["k_cmp"], inp["v_cmp"], inp["scores"], center=True)
    assert np.abs(got - expect).max() < 1e-12


@pytest.mark.parametrize("center", [False, True], ids=["token", "centre"])
def test_summaries_with_origin_use_true_coordinates(center):
    # Both summary forms of a sub-volume whose first plane is true plane 9: the rotation
    # before pooling (Key design 2) and the centre variant both see origin + local coordinate.
    origin = (9, 0, 0)
    s = small(Z=4, origin=origin)
    inp, g2p, mem = _summary_case(s, seed=8)
    coords = inp["coords"].numpy()
    kc, sc = oracle.as_f64(inp["k_cmp"]), oracle.as_f64(inp["scores"])
    a = scipy.special.softmax(sc[mem], axis=1)                               # [M, v, Hkv]
    if center:
        expect = rope_complex(s, _block_centres(s) + np.asarray(origin), np.einsum("jug,jugd->jgd", a, kc[mem]))
    else:
        kr = rope_complex(s, coords + np.asarray(origin), kc)
        expect = np.einsum("jug,jugd->jgd", a, kr[mem])
    got, vs = oracle.summaries(s, coords, mem, inp["k_cmp"], inp["v_cmp"], inp["scores"], center=center)
    assert np.abs(got - expect).max() < 1e-12
    _, vs0 = oracle.summaries(s.replace(origin=(0, 0, 0)), coords, mem, inp["k_cmp"], inp["v_cmp"],
                              inp["scores"], center=center)
    assert np.abs(vs - vs0).max() == 0                                          # values carry no rotation


def test_summary_center_error_within_rotation_bound():
    # Per plane ||R(t1) - R(t2)|| = 2 |sin((t1 - t2) / 2)|, so the key difference of the two
    # variants is at most sum_u a_u * max_p 2|sin(omega_p (cbar - c_u)_axis(p) / 2)| * ||k_u||.
    s = small(Z=2, H=8, W=8)
    inp, g2p, mem = _summary_case(s, seed=9)
    coords = inp["coords"].numpy()
    kt, _ = oracle.summaries(s, coords, mem, inp["k_cmp"], inp["v_cmp"], inp["scores"])
    kc, _ = oracle.summaries(s, coords, mem, inp["k_cmp"], inp["v_cmp"], inp["scores"], center=True)
    a = scipy.special.softmax(oracle.as_f64(inp["scores"])[mem], axis=1)
    knorm = np.linalg.norm(oracle.as_f64(inp["k_cmp"])[mem], axis=-1)          # [M, v, Hkv]
    omegas = [s.rope_base ** (-np.arange(m) / m) for m in (s.m_z, s.m_y, s.m_x)]
    delta = _block_centres(s)[:, None, :] - coords[mem].astype(np.float64)       # [M, v, 3]
    bound_u = np.max(np.stack([np.max(2 * np.abs(np.sin(om[None, None, :] * delta[..., ax:ax + 1] / 2)), axis=-1)
                               for ax, om in enumerate(omegas)]), axis=0)          # [M, v]
    bound = np.einsum("jug,ju,jug->jg", a, bound_u, knorm)
    diff = np.linalg.norm(kc - kt, axis=-1)
    assert (diff <= bound + 1e-12).all()
    assert diff.max() > 1e-3          # an approximation, not the identity


# ----------------------------------------------------------- branches -------

def _lattice_dist_mask(coords_q, coords_k, s):
    d = np.abs(coords_q[:, None, :].astype(np.int64) - coords_k[None, :, :].astype(np.int64))
    return (d[..., 0] <= s.rz) & (d[..., 1] <= s.ry) & (d[..., 2] <= s.rx)


@pytest.mark.parametrize("packing", ["raster", "random"])
def test_local_branch_equals_masked_dense_attention(packing):
    s = small()
    inp = synth.make_inputs(s, packing, 5)
    coords = inp["coords"].numpy()
    st, g2p, mem = oracle.build_index(s, coords)
    qr = rope_complex(s, coords, oracle.as_f64(inp["q"]))
    kr = rope_complex(s, coords, oracle.as_f64(inp["k_loc"]))
    o = oracle.local_attn(s, coords, g2p, qr, kr, inp["v_loc"])
    mask = _lattice_dist_mask(coords, coords, s)
    ref = sdpa64(qr, expand_kv(s, kr), expand_kv(s, oracle.as_f64(inp["v_loc"])),
                 s.softmax_scale, mask[None])
    assert np.abs(o - ref).max() < 1e-12


def test_whole_volume_window_gate_local_is_dense_rope_attention():
    # Window covering the volume + gate pinned to the local branch = dense attention
    # with 3D RoPE (the local branch is exact).
    s = small(Z=2, H=4, W=8, rz=2, ry=4, rx=8)
    inp = synth.make_inputs(s, "morton", 6)
    inp["gate"][..., 0] = 1e4
    inp["gate"][..., 1] = -1e4
    res = oracle.forward(s, inp)
    coords = inp["coords"].numpy()
    qr = rope_complex(s, coords, oracle.as_f64(inp["q"]))
    kr = rope_complex(s, coords, oracle.as_f64(inp["k_loc"]))
    ref = sdpa64(qr, expand_kv(s, kr), expand_kv(s, oracle.as_f64(inp["v_loc"])), s.softmax_scale)
    assert np.abs(res["out"] - ref).max() < 1e-12


def test_unit_blocks_gate_compressed_is_dense_attention_on_cmp():
    s = small(by=1, bx=1)
    inp = synth.make_inputs(s, "block", 7)
    inp["gate"][..., 0] = -1e4
    inp["gate"][..., 1] = 1e4
    res = oracle.forward(s, inp)
    coords = inp["coords"].numpy()
    qr = rope_complex(s, coords, oracle.as_f64(inp["q"]))
    kr = rope_complex(s, coords, oracle.as_f64(inp["k_cmp"]))
    ref = sdpa64(qr, expand_kv(s, kr), expand_kv(s, oracle.as_f64(inp["v_cmp"])), s.softmax_scale)
    assert np.abs(res["out"] - ref).max() < 1e-12


def test_compressed_branch_is_sdpa_over_summaries():
    s = small()
    inp = synth.make_inputs(s, "random", 8)
    res = oracle.forward(s, inp)
    ref = sdpa64(res["q_rot"], expand_kv(s, res["k_sum"]), expand_kv(s, res["v_sum"]),
                 s.softmax_scale)
    assert np.abs(res["o_cmp"] - ref).max() < 1e-12


def test_gate_is_two_way_softmax():
    s = small()
    inp = synth.make_inputs(s, "raster", 9)
    res = oracle.forward(s, inp)
    w = torch.softmax(inp["gate"].double(), dim=-1).numpy()
    ref = w[..., 0:1] * res["o_loc"] + w[..., 1:2] * res["o_cmp"]
    assert np.abs(res["out"] - ref).max() < 1e-14
    zero = {**inp, "gate": torch.zeros_like(inp["gate"])}
    r0 = oracle.forward(s, zero)
    assert np.abs(r0["out"] - 0.5 * (r0["o_loc"] + r0["o_cmp"])).max() < 1e-15


# ------------------------------------------------------- whole operator -----

@pytest.mark.parametrize("shape", [TINY, small(Z=2, H=8, W=12, rz=1, ry=3, rx=3)])
def test_proposition_1_packing_equivariance(shape):
    # A(PX, Pc) = P A(X, c) for coordinate-preserving repackings (Key design 1).
    sv = synth.draw_site_values(shape, 11)
    ref = oracle.forward(shape, synth.make_inputs(shape, "raster", 11, sv))["out"]
    for p in ("morton", "block", "random"):
        inp = synth.make_inputs(shape, p, 11, sv)
        out = oracle.forward(shape, inp)["out"]
        sites = inp["sites"].numpy()
        assert np.abs(out - ref[sites]).max() < 1e-12, p


def test_packed_index_rope_breaks_equivariance():
    # Negative control: RoPE on the packed index (a 1-D coordinate) is not
    # packing-equivariant, so the test above has power.
    s = TINY
    sv = synth.draw_site_values(s, 12)

    def packed_rope_forward(inp):
        coords = inp["coords"].numpy()
        fake = np.zeros_like(coords)
        fake[:, 2] = np.arange(s.N)
        st, g2p, mem = oracle.build_index(s, coords)
        qr = oracle.rotate(s, fake, inp["q"])
        kr = oracle.rotate(s, fake, inp["k_loc"])
        ks, vs = oracle.summaries(s, fake, mem, inp["k_cmp"], inp["v_cmp"], inp["scores"])
        ol = oracle.local_attn(s, coords, g2p, qr, kr, inp["v_loc"])
        oc = oracle.summary_attn(s, qr, ks, vs)
        return oracle.gate_mix(s, inp["gate"], ol, oc)

    ref = packed_rope_forward(synth.make_inputs(s, "raster", 12, sv))
    inp = synth.make_inputs(s, "random", 12, sv)
    out = packed_rope_forward(inp)
    assert np.abs(out - ref[inp["sites"].numpy()]).max() > 1e-2


def test_translation_invariance():
    # Logits depend only on displacements: shifting every coordinate used by the
    # rotation leaves the output unchanged.
    s = small()
    inp = synth.make_inputs(s, "random", 13)
    coords = inp["coords"].numpy()
    base = oracle.forward(s, inp)
    sh = coords + np.array([5, -17, 101], np.int32)
    qr = oracle.rotate(s, sh, inp["q"])
    kr = oracle.rotate(s, sh, inp["k_loc"])
    ks, vs = oracle.summaries(s, sh, base["members"], inp["k_cmp"], inp["v_cmp"], inp["scores"])
    ol = oracle.local_attn(s, coords, base["g2p"], qr, kr, inp["v_loc"])
    oc = oracle.summary_attn(s, qr, ks, vs)
    out = oracle.gate_mix(s, inp["gate"], ol, oc)
    assert np.abs(out - base["out"]).max() < 1e-12


def test_sampled_rows_match_full_run():
    s = TINY
    inp = synth.make_inputs(s, "random", 14)
    full = oracle.forward(s, inp)
    rows = synth.sample_rows(s.N, 17, 3)
    part = oracle.forward(s, inp, rows)
    assert np.array_equal(part["out"], full["out"][rows])


def test_page_printed_shape_facts():
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "page_shape_facts.json")
    facts = json.load(open(path))
    for f in facts["facts"]:
        assert math.prod(f["factors"]) == f["value"], f["what"]
    for r in facts["ratios"]:
        assert round(r["num"] / r["den"], r["digits"]) == r["value"], r["what"]
    s = synth.CONFIGS["262k"]
    assert s.N * s.M == facts["facts"][0]["value"] and s.M * s.v == s.N
    assert 2 * (s.m_z + s.m_y + s.m_x) == s.d_h
