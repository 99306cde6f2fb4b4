"""The z-slab split of one volume over several ranks, host logic on CPU gloo ranks.

Each rank takes the tokens of its planes, exchanges its boundary planes' local
keys and values with its neighbours, and runs the stages on its slab extended
by the received halo, a lattice whose origin is the true z of its first plane.
Here the stages are the oracle's (float64, CPU), the exchanges are gloo's, and
the arrangement of tensors (which rows are sent, how the extended lattice is
laid out, which summaries are a rank's own, how the gathered summaries are
ordered) is the library's own z-slab module.  Every rank's outputs must equal
the whole-volume oracle's for the same tokens (the local window of a boundary
query, the summaries of every block and the rotation of every token depend on
all of it being right), and the index map and block membership of its own
planes, mapped to whole-volume token ids, must equal the whole volume's bit
for bit.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shape(**kw):
    import synth
    base = dict(Z=7, H=8, W=12, Hq=4, Hkv=2, bz=1, by=2, bx=4, rz=2, ry=2, rx=3, dtype="f32",
                value_scale=1.0, packing="random")
    base.update(kw)
    return synth.Pack3DShape(**base)


def _rank(rank, world, port, shape_kw, center, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle
    import synth
    from geometry_aware_local_b200 import zslab
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        s = _shape(**shape_kw)
        inp = synth.make_inputs(s, seed=41)
        whole = oracle.forward(s, inp, center=center)
        p = zslab.make_plan(s, rank, world)
        idx, own = zslab.take_slab(inp, p)
        below, above = zslab.exchange_halo(own["k_loc"], own["v_loc"], own["coords"], p)
        ext = zslab.prepare(own, below, above, p)
        se = s.replace(Z=p.Z_ext, origin=(s.origin[0] + p.z0 - p.lo, s.origin[1], s.origin[2]))
        st, g2p, mem = oracle.build_index(se, ext["coords"])
        assert st == 0
        coords = ext["coords"].numpy()
        # The index map and block membership of the rank's own planes, mapped to whole-volume
        # token ids (own tokens through take_slab's indices, halo tokens through their true
        # coordinates), must be the whole volume's, bit for bit.
        st_w, g2p_w, mem_w = oracle.build_index(s, inp["coords"])
        true_z = coords[:, 0] + (p.z0 - p.lo)
        ext2glob = g2p_w[(true_z * s.H + coords[:, 1]) * s.W + coords[:, 2]].astype(np.int64)
        ext2glob[:p.tokens] = idx.numpy()
        hw, bpp = s.H * s.W, (s.H // s.by) * (s.W // s.bx)
        index_exact = bool(np.array_equal(ext2glob[g2p[p.lo * hw:(p.lo + p.planes) * hw]],
                                          g2p_w[p.z0 * hw:p.z1 * hw]) and
                           np.array_equal(ext2glob[mem[p.lo * bpp:(p.lo + p.planes) * bpp]],
                                          mem_w[p.z0 * bpp:p.z1 * bpp]))
        rows = np.arange(p.tokens)
        qr = oracle.rotate(se, coords[:p.tokens], ext["q"][:p.tokens])
        kr = oracle.rotate(se, coords, ext["k_loc"])
        ks, vs = oracle.summaries(se, coords, mem, ext["k_cmp"], ext["v_cmp"], ext["scores"], center=center)
        ol = oracle.local_attn(se, coords, g2p, qr, kr, ext["v_loc"].numpy(), rows)
        k_own, v_own = zslab.own_summaries(torch.from_numpy(ks), torch.from_numpy(vs), p, bpp)
        k_all, v_all = zslab.gather_summaries(k_own, v_own, p, bpp)
        oc = oracle.summary_attn(se, qr, k_all.numpy(), v_all.numpy())
        out = oracle.gate_mix(se, ext["gate"].numpy(), ol, oc, rows)
        ref = whole["out"][idx.numpy()]
        q.put((rank, float(np.abs(out - ref).max() / np.abs(ref).max()),
               float(np.abs(ol - whole["o_loc"][idx.numpy()]).max()),
               float(max(np.abs(k_all.numpy() - whole["k_sum"]).max(), np.abs(v_all.numpy() - whole["v_sum"]).max())),
               p.lo, p.hi, index_exact, None))
    except Exception as e:                       # report instead of hanging the parent
        q.put((rank, None, None, None, None, None, None, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


def _run(world, shape_kw=None, center=False):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, shape_kw or {}, center, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=240) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
    for rank, *_, err in got:
        assert err is None, f"rank {rank}: {err}"
    assert all(p.exitcode == 0 for p in procs)
    return got


@pytest.mark.parametrize("world", [2, 3])
def test_zslab_ranks_equal_whole_volume(world):
    got = _run(world)
    for rank, out_err, loc_err, sum_err, lo, hi, index_exact, _ in got:
        assert lo == (0 if rank == 0 else 2) and hi == (0 if rank == world - 1 else 2)
        assert index_exact, rank
        assert out_err < 1e-12, (rank, out_err)
        assert loc_err < 1e-12, (rank, loc_err)
        assert sum_err < 1e-12, (rank, sum_err)


def test_zslab_centre_variant_and_shifted_volume():
    # The summary-centre variant, and a volume that itself starts at a nonzero origin.
    got = _run(2, dict(origin=(5, 2, 0), rz=1), center=True)
    for rank, out_err, loc_err, sum_err, lo, hi, index_exact, _ in got:
        assert out_err < 1e-12 and loc_err < 1e-12 and sum_err < 1e-12 and index_exact, rank


# ------------------------------------------------------------- host plan -----

def test_slab_bounds_and_plan():
    from geometry_aware_local_b200 import zslab
    assert zslab.slab_bounds(7, 3) == [(0, 3), (3, 5), (5, 7)]
    assert zslab.slab_bounds(16, 1) == [(0, 16)]
    s = _shape(Z=16)
    p = zslab.make_plan(s, 1, 4)
    assert (p.z0, p.z1, p.lo, p.hi, p.Z_ext, p.tokens) == (4, 8, 2, 2, 8, 4 * 8 * 12)
    p0 = zslab.make_plan(s, 0, 1)
    assert (p0.lo, p0.hi, p0.Z_ext) == (0, 0, 16)
    with pytest.raises(ValueError):
        zslab.make_plan(s.replace(bz=2), 0, 2)            # a block would straddle two slabs
    with pytest.raises(ValueError):
        zslab.make_plan(s.replace(rz=5), 0, 4)            # slabs of 4 planes, halo of 5
    with pytest.raises(ValueError):
        zslab.slab_bounds(3, 4)


def test_boundary_rows_are_raster_planes():
    import synth
    from geometry_aware_local_b200 import zslab
    s = _shape(Z=4)
    inp = synth.make_inputs(s, seed=3)
    p = zslab.make_plan(s, 0, 1)
    first, last = zslab.boundary_rows(inp["coords"], p)
    c = inp["coords"][first]
    n = s.rz * s.H * s.W
    want = np.stack(np.meshgrid(np.arange(s.rz), np.arange(s.H), np.arange(s.W), indexing="ij"), -1).reshape(n, 3)
    assert np.array_equal(c.numpy(), want)
    assert np.array_equal(inp["coords"][last].numpy(), want + np.array([s.Z - s.rz, 0, 0]))


def test_ext_config_shifts_origin_and_keeps_everything_else():
    import geometry_aware_local_b200 as p3
    from geometry_aware_local_b200 import zslab
    cfg = p3.make_config(16, 8, 12, block=(1, 2, 4), radius=(2, 2, 3), origin=(3, 1, 0))
    p = zslab.make_plan(cfg, 2, 4)
    e = zslab.ext_config(cfg, p)
    assert (e.Z, list(e.origin)) == (8, [3 + 8 - 2, 1, 0])
    assert (cfg.Z, list(cfg.origin)) == (16, [3, 1, 0])      # the caller's config is untouched
    assert p3.validate(e) == 0 and (e.H, e.W, e.rz, e.by, e.bx) == (8, 12, 2, 2, 4)
