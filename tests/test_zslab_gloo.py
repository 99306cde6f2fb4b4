"""The z-slab split of one volume over several ranks, host logic on CPU gloo ranks.

(The last group of tests below runs zslab.Plan's own exchange code on gloo ranks.)

Each rank takes the tokens of its planes, exchanges its boundary planes' local
keys and values with its neighbours, and runs the stages on its slab extended
by the received halo, a lattice whose origin is the true z of its first plane.
Here the stages are the oracle's (float64, CPU), the exchanges are gloo's, and
the layout is the library's z-slab module's (the extended lattice's
coordinates and rows, which index-map slice is sent and where the halo lands,
which summaries each rank contributes to the all-gather and which of them are
kept); the row movement itself, done on the GPU by pack3d_gather_rows and
NCCL, is done here by CPU indexing.  Every rank's outputs must equal
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

NAMES = ("coords", "q", "k_loc", "v_loc", "k_cmp", "v_cmp", "scores", "gate")

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
        st_w, g2p_w, mem_w = oracle.build_index(s, inp["coords"])
        p = zslab.make_plan(s, rank, world)
        idx, own = zslab.take_slab(inp, p)
        # The extended lattice as zslab.Plan lays it out: own rows, then the halo planes.
        coords = zslab.ext_coords(own["coords"], p).numpy()
        se = s.replace(Z=p.Z_ext, origin=(s.origin[0] + p.z0 - p.lo, s.origin[1], s.origin[2]))
        st, g2p, mem = oracle.build_index(se, coords)
        assert st == 0
        N_e = p.Z_ext * s.H * s.W
        ext = {k: torch.zeros((N_e,) + tuple(own[k].shape[1:]), dtype=own[k].dtype) for k in NAMES if k != "coords"}
        for k in ext:
            ext[k][:p.tokens] = own[k]
        # The index map and block membership of the rank's own planes, mapped to whole-volume
        # token ids (own tokens through take_slab's indices, halo tokens through their true
        # coordinates), must be the whole volume's, bit for bit.
        true_z = coords[:, 0] + (p.z0 - p.lo)
        ext2glob = g2p_w[(true_z * s.H + coords[:, 1]) * s.W + coords[:, 2]].astype(np.int64)
        ext2glob[:p.tokens] = idx.numpy()
        hw, bpp = s.H * s.W, (s.H // s.by) * (s.W // s.bx)
        index_exact = bool(np.array_equal(ext2glob[g2p[p.lo * hw:(p.lo + p.planes) * hw]],
                                          g2p_w[p.z0 * hw:p.z1 * hw]) and
                           np.array_equal(ext2glob[mem[p.lo * bpp:(p.lo + p.planes) * bpp]],
                                          mem_w[p.z0 * bpp:p.z1 * bpp]))
        # Halo: the boundary planes' rows (index-map slices, raster order) to the neighbours,
        # theirs into the halo rows.
        ops = []
        for peer, (a, b), (ra, rb), n in ((rank - 1, p.send_below, p.halo_below, p.lo),
                                          (rank + 1, p.send_above, p.halo_above, p.hi)):
            if n:
                rows = torch.from_numpy(g2p[a:b].astype(np.int64))
                for name in ("k_loc", "v_loc"):
                    ops.append(dist.P2POp(dist.isend, ext[name].index_select(0, rows).contiguous(), peer))
                    ops.append(dist.P2POp(dist.irecv, ext[name][ra:rb], peer))
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()
        rows = np.arange(p.tokens)
        qr = oracle.rotate(se, coords[:p.tokens], ext["q"][:p.tokens])
        kr = oracle.rotate(se, coords, ext["k_loc"])
        ks, vs = oracle.summaries(se, coords, mem, ext["k_cmp"], ext["v_cmp"], ext["scores"], center=center)
        ol = oracle.local_attn(se, coords, g2p, qr, kr, ext["v_loc"].numpy(), rows)
        # Summaries: every rank's part (summary_parts), all-gathered, then the own blocks kept.
        parts = zslab.summary_parts(s, world)
        start, _, _ = parts[rank]
        most = max(c for _, _, c in parts)
        got = []
        for arr in (ks, vs):
            part = torch.from_numpy(np.ascontiguousarray(arr[start:start + most]))
            bufs = [torch.empty_like(part) for _ in range(world)]
            dist.all_gather(bufs, part)
            got.append(np.concatenate([bufs[r].numpy()[o:o + c] for r, (_, o, c) in enumerate(parts)]))
        k_all, v_all = got
        oc = oracle.summary_attn(se, qr, k_all, v_all)
        out = oracle.gate_mix(se, ext["gate"].numpy(), ol, oc, rows)
        ref = whole["out"][idx.numpy()]
        q.put((rank, float(np.abs(out - ref).max() / np.abs(ref).max()),
               float(np.abs(ol - whole["o_loc"][idx.numpy()]).max()),
               float(max(np.abs(k_all - whole["k_sum"]).max(), np.abs(v_all - whole["v_sum"]).max())),
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


# ------------------------------------------------- zslab.Plan on gloo ranks -----
#
# zslab.Plan itself on CPU gloo ranks: its buffers, its index-map slices, its halo
# exchange (batch_isend_irecv) and its summary all-gather (all_gather_into_tensor,
# then the compaction for uneven slabs) run as written; only the library's kernel
# calls are replaced, for this test, by the oracle's stages on the extended
# lattice (and the row gather by CPU indexing).  The outputs must equal the
# whole-volume oracle's, the halo rows the neighbours' boundary planes bit for
# bit, and the gathered summaries the whole volume's.

def _install_oracle_stand_ins(p3, se, state):
    """Replaces the binding's kernel calls the Plan makes by the oracle's stages on the extended
    lattice `se` (test infrastructure; the product path never calls the oracle)."""
    import oracle

    def build_index(cfg, coords, g2p, members, err, stream=None):
        assert (cfg.Z, tuple(cfg.origin)) == (se.Z, tuple(se.origin))   # the Plan's extended config
        st, g, m = oracle.build_index(se, coords.numpy())
        assert st == 0
        g2p.copy_(torch.from_numpy(g))
        members.copy_(torch.from_numpy(m))
        state["coords"] = coords.numpy().copy()

    def build_summaries(cfg, members, k_cmp, v_cmp, scores, k_sum, v_sum, stream=None):
        ks, vs = oracle.summaries(se, state["coords"], members, k_cmp, v_cmp, scores)
        k_sum.copy_(torch.from_numpy(ks))
        v_sum.copy_(torch.from_numpy(vs))

    def rope_qk(cfg, coords, q, q_rot, k, k_rot, stream=None):
        q_rot.copy_(torch.from_numpy(oracle.rotate(se, coords, q)))
        k_rot.copy_(torch.from_numpy(oracle.rotate(se, coords, k)))

    def local_attn(cfg, g2p, q_rot, k_rot, v_loc, o_loc, err=None, stream=None):
        t = state["tokens"]   # the own rows come first in the extended layout
        o = oracle.local_attn(se, state["coords"], g2p, q_rot[:t], k_rot, v_loc, np.arange(t))
        o_loc[:t].copy_(torch.from_numpy(o))

    def summary_attn_rows(cfg, tokens, summaries, q_rot, k_sum, v_sum, o_loc, gate, out, err=None, stream=None):
        assert k_sum.shape[0] == summaries and q_rot.shape[0] == tokens
        oc = oracle.summary_attn(se, q_rot, k_sum, v_sum)
        out.copy_(torch.from_numpy(oracle.gate_mix(se, gate, o_loc, oc, np.arange(tokens))))

    def gather_rows(idx, src, dst, stream=None):
        i = idx.long()
        rows = src.index_select(0, i.clamp(min=0))
        rows[i < 0] = 0
        dst.copy_(rows)

    def check_status(err, stream=None):
        return int(err.abs().sum())

    for name, fn in (("build_index", build_index), ("build_summaries", build_summaries), ("rope_qk", rope_qk),
                     ("local_attn", local_attn), ("summary_attn_rows", summary_attn_rows),
                     ("gather_rows", gather_rows), ("check_status", check_status)):
        setattr(p3, name, fn)


def _plan_rank(rank, world, port, shape_kw, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import geometry_aware_local_b200 as p3
    import oracle
    import synth
    from geometry_aware_local_b200 import zslab
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        s = _shape(**shape_kw)
        inp = synth.make_inputs(s, seed=43)
        whole = oracle.forward(s, inp)
        _, g2p_w, _ = oracle.build_index(s, inp["coords"])
        cfg = p3.config_from_shape(s)
        p = zslab.make_plan(cfg, rank, world)
        se = s.replace(Z=p.Z_ext, origin=(s.origin[0] + p.z0 - p.lo, s.origin[1], s.origin[2]))
        _install_oracle_stand_ins(p3, se, {"tokens": p.tokens})
        idx, own = zslab.take_slab(inp, p)
        plan = zslab.Plan(cfg, own["coords"], rank, world)
        for k, v in plan.inputs().items():
            v.copy_(own[k])
        out = plan.forward().double().numpy()
        ref = whole["out"][idx.numpy()]
        out_err = float(np.abs(out - ref).max() / np.abs(ref).max())
        # The halo rows: the neighbours' boundary planes in raster order, bit for bit.
        hw = s.H * s.W
        halo_exact = True
        for (a, b), z_from in ((p.halo_below, p.z0 - p.lo), (p.halo_above, p.z1)):
            if b > a:
                tok = torch.from_numpy(g2p_w[z_from * hw:z_from * hw + (b - a)].astype(np.int64))
                for name in ("k_loc", "v_loc"):
                    halo_exact = halo_exact and torch.equal(plan.ext[name][a:b], inp[name].index_select(0, tok))
        k_err = max(float(np.abs(plan.k_all.double().numpy() - whole["k_sum"]).max() / np.abs(whole["k_sum"]).max()),
                    float(np.abs(plan.v_all.double().numpy() - whole["v_sum"]).max() / np.abs(whole["v_sum"]).max()))
        q.put((rank, out_err, k_err, halo_exact, plan.uneven, p.lo, p.hi, None))
    except Exception as e:                       # report instead of hanging the parent
        q.put((rank, None, None, None, None, None, None, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,Z,uneven", [(2, 8, False), (2, 7, True), (3, 7, True)])
def test_plan_exchanges_on_gloo_ranks(world, Z, uneven):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_plan_rank, args=(r, world, port, dict(Z=Z), q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=240) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
    for rank, *_, err in got:
        assert err is None, f"rank {rank}: {err}"
    assert all(p.exitcode == 0 for p in procs)
    for rank, out_err, k_err, halo_exact, was_uneven, lo, hi, _ in got:
        assert (lo > 0) == (rank > 0) and (hi > 0) == (rank < world - 1), rank
        assert was_uneven == uneven, rank
        assert halo_exact, rank
        # float32 buffers between the oracle's float64 stages
        assert out_err < 1e-5, (rank, out_err)
        assert k_err < 1e-6, (rank, k_err)


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


def test_layout_ranges_and_summary_parts():
    from geometry_aware_local_b200 import zslab
    s = _shape(Z=7)                       # 4 + 3 planes over two ranks, 8 x 12 sites per plane, rz = 2
    p0, p1 = zslab.make_plan(s, 0, 2), zslab.make_plan(s, 1, 2)
    hw = s.H * s.W
    # rank 0: own planes 0-3 (rows 0 .. 4hw), halo above = true planes 4-5 after them
    assert (p0.lo, p0.hi, p0.Z_ext) == (0, 2, 6)
    assert p0.halo_below == (4 * hw, 4 * hw) and p0.halo_above == (4 * hw, 6 * hw)
    assert p0.send_above == (2 * hw, 4 * hw)           # its last two planes, extended-lattice sites
    # rank 1: halo below = true planes 2-3 (extended planes 0-1), own planes 4-6 (extended 2-4)
    assert (p1.lo, p1.hi, p1.Z_ext) == (2, 0, 5)
    assert p1.halo_below == (3 * hw, 5 * hw) and p1.halo_above == (5 * hw, 5 * hw)
    assert p1.send_below == (2 * hw, 4 * hw)
    # summaries: 4 and 3 planes of 4 x 3 blocks; rank 1's part reaches back into its halo blocks
    bpp = (s.H // s.by) * (s.W // s.bx)
    assert zslab.summary_parts(s, 2) == [(0, 0, 4 * bpp), (1 * bpp, 1 * bpp, 3 * bpp)]
    even = zslab.summary_parts(_shape(Z=8), 2)
    assert all(o == 0 and c == 4 * bpp for _, o, c in even)
    ext = zslab.ext_coords(torch.zeros((p1.tokens, 3), dtype=torch.int32), p1)
    assert ext.shape == (p1.Z_ext * hw, 3)
    assert ext[:p1.tokens, 0].eq(2).all()                 # own z shifted by lo
    assert ext[p1.tokens:, 0].tolist() == [z for z in (0, 1) for _ in range(hw)]


def test_ext_config_shifts_origin_and_keeps_everything_else():
    import geometry_aware_local_b200 as p3
    from geometry_aware_local_b200 import zslab
    cfg = p3.make_config(16, 8, 12, block=(1, 2, 4), radius=(2, 2, 3), origin=(3, 1, 0))
    p = zslab.make_plan(cfg, 2, 4)
    e = zslab.ext_config(cfg, p)
    assert (e.Z, list(e.origin)) == (8, [3 + 8 - 2, 1, 0])
    assert (cfg.Z, list(cfg.origin)) == (16, [3, 1, 0])      # the caller's config is untouched
    assert p3.validate(e) == 0 and (e.H, e.W, e.rz, e.by, e.bx) == (8, 12, 2, 2, 4)
