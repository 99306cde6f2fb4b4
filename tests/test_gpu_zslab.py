"""The z-slab split of one volume on one GPU: every rank's steps, in turn, in one process.

No rank waits on another here: the halo planes and the gathered summaries are
handed from one rank's tensors to the next by indexing, where the
distributed path sends them (the gloo tests cover that host logic).  Each rank
runs the library's kernels on its extended lattice, whose origin is the true z
of its first plane; the concatenation of all ranks' outputs must match the
whole-volume call: summaries and rotated queries bit for bit (the same
arithmetic at the same true coordinates), the local branch and the output
within the parity tolerance of the float64 oracle, and against the
whole-volume kernels within float accumulation-order rounding.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


@pytest.fixture(scope="module")
def p3(cuda_device):
    import geometry_aware_local_b200 as p3
    return p3


def rel_err(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(gpu - ref).max() / max(np.abs(ref).max(), 1e-30))


def whole_volume(p3, cfg, s, d):
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    g2p = torch.empty(s.N, dtype=torch.int32, device="cuda")
    mem = torch.empty(s.M, s.v, dtype=torch.int32, device="cuda")
    p3.build_index(cfg, d["coords"], g2p, mem, err)
    ks = torch.empty(s.M, s.Hkv, s.d_h, dtype=d["q"].dtype, device="cuda")
    vs = torch.empty_like(ks)
    p3.build_summaries(cfg, mem, d["k_cmp"], d["v_cmp"], d["scores"], ks, vs)
    qr, kr = torch.empty_like(d["q"]), torch.empty_like(d["k_loc"])
    p3.rope_qk(cfg, d["coords"], d["q"], qr, d["k_loc"], kr)
    ol = torch.empty(s.N, s.Hq, s.d_h, dtype=torch.float32, device="cuda")
    p3.local_attn(cfg, g2p, qr, kr, d["v_loc"], ol, err)
    out = torch.empty_like(d["q"])
    p3.summary_attn(cfg, qr, ks, vs, ol, d["gate"], out, err)
    assert p3.check_status(err) == 0
    return dict(k_sum=ks, v_sum=vs, q_rot=qr, o_loc=ol, out=out)


def emulate(p3, cfg, s, d, world):
    """Every rank's phases on this GPU; returns the whole-volume arrays assembled from the ranks."""
    from geometry_aware_local_b200 import zslab
    plans = [zslab.make_plan(cfg, r, world) for r in range(world)]
    takes = [zslab.take_slab(d, p) for p in plans]
    edges = [zslab.boundary_rows(own["coords"], p) for p, (_, own) in zip(plans, takes)]
    kv = [torch.stack([own["k_loc"], own["v_loc"]], dim=1) for _, own in takes]
    none = kv[0][:0]
    bpp = (cfg.H // cfg.by) * (cfg.W // cfg.bx)
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    ranks = []
    for r, p in enumerate(plans):
        below = kv[r - 1][edges[r - 1][1]] if p.lo else none      # the last rz planes of the rank below
        above = kv[r + 1][edges[r + 1][0]] if p.hi else none      # the first rz planes of the rank above
        ext = zslab.prepare(takes[r][1], below, above, p)
        cfg_e = zslab.ext_config(cfg, p)
        q_rot, o_loc, k_sum, v_sum = zslab.local_stage(cfg_e, ext, err)
        ranks.append((cfg_e, ext, q_rot, o_loc) + tuple(zslab.own_summaries(k_sum, v_sum, p, bpp)))
    k_all = torch.cat([rk[4] for rk in ranks])
    v_all = torch.cat([rk[5] for rk in ranks])
    res = dict(k_sum=k_all, v_sum=v_all, q_rot=torch.empty_like(d["q"]), out=torch.empty_like(d["q"]),
               o_loc=torch.empty(s.N, s.Hq, s.d_h, dtype=torch.float32, device="cuda"))
    for p, (idx, _), (cfg_e, ext, q_rot, o_loc, _, _) in zip(plans, takes, ranks):
        out = zslab.global_stage(cfg_e, p.tokens, q_rot, k_all, v_all, o_loc, ext["gate"], err)
        res["out"][idx] = out
        res["q_rot"][idx] = q_rot[:p.tokens]
        res["o_loc"][idx] = o_loc[:p.tokens]
    assert p3.check_status(err) == 0
    return res


CASES = {
    "ragged-w2": (synth.Pack3DShape(Z=7, H=12, W=20, Hq=8, Hkv=2, rz=2, ry=3, rx=3, dtype="bf16",
                                    value_scale=0.125, packing="random"), 2, 0),
    "ragged-w3-f32": (synth.Pack3DShape(Z=7, H=12, W=20, Hq=8, Hkv=2, rz=2, ry=3, rx=3, dtype="f32",
                                        value_scale=1.0, packing="random"), 3, 0),
    "centre-w2": (synth.Pack3DShape(Z=6, H=16, W=16, Hq=8, Hkv=2, rz=1, ry=3, rx=3, dtype="bf16",
                                    value_scale=0.125, packing="morton", origin=(4, 0, 0)), 2, 0x4),
    "65k-w2": (synth.CONFIGS["65k"], 2, 0),
    "65k-w8": (synth.CONFIGS["65k"], 8, 0),
}


@pytest.mark.parametrize("name", list(CASES))
def test_zslab_emulated_ranks_match_whole_volume(p3, name):
    s, world, flags = CASES[name]
    inp = synth.make_inputs(s, seed=51)
    d = {k: v.cuda() for k, v in inp.items() if k != "sites"}
    cfg = p3.config_from_shape(s, flags)
    whole = whole_volume(p3, cfg, s, d)
    got = emulate(p3, cfg, s, d, world)
    for k in ("k_sum", "v_sum", "q_rot"):
        assert torch.equal(got[k], whole[k]), k
    assert rel_err(got["o_loc"].cpu(), whole["o_loc"].cpu()) <= 1e-5
    assert rel_err(got["out"].float().cpu(), whole["out"].float().cpu()) <= (1e-5 if s.dtype == "f32" else 1e-2)
    rows = np.random.default_rng(7).choice(s.N, size=min(s.N, 384), replace=False)
    ref = oracle.forward(s, inp, rows=rows, center=bool(flags & 0x4))
    assert rel_err(got["out"].float().cpu().numpy()[rows], ref["out"]) <= TOL[s.dtype]
    assert rel_err(got["o_loc"].cpu().numpy()[rows], ref["o_loc"]) <= TOL[s.dtype]


def test_summary_attn_rows_on_a_subset_of_rows(p3):
    """pack3d_summary_attn_rows: a prefix of the queries against summaries of another count."""
    s = synth.Pack3DShape(Z=3, H=16, W=16, Hq=8, Hkv=2, dtype="bf16", value_scale=0.125)
    inp = synth.make_inputs(s, seed=52)
    d = {k: v.cuda() for k, v in inp.items() if k != "sites"}
    cfg = p3.config_from_shape(s)
    whole = whole_volume(p3, cfg, s, d)
    extra = (torch.randn(40, s.Hkv, s.d_h, device="cuda") * 0.125).to(torch.bfloat16)
    k_all = torch.cat([whole["k_sum"], extra])
    v_all = torch.cat([whole["v_sum"], extra.flip(0)])
    n = 333                                               # ragged: not a multiple of the query tile
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    out = torch.empty(n, s.Hq, s.d_h, dtype=torch.bfloat16, device="cuda")
    p3.summary_attn_rows(cfg, n, k_all.shape[0], whole["q_rot"][:n], k_all, v_all, whole["o_loc"][:n],
                         d["gate"][:n], out, err)
    assert p3.check_status(err) == 0
    qr = whole["q_rot"][:n].cpu()
    oc = oracle.summary_attn(s, qr, k_all.cpu(), v_all.cpu())
    ref = oracle.gate_mix(s, d["gate"].cpu(), whole["o_loc"][:n].cpu(), oc, np.arange(n))
    assert rel_err(out.float().cpu().numpy(), ref) <= TOL["bf16"]
    # zero tokens: nothing to do, nothing written
    before = out.clone()
    p3.summary_attn_rows(cfg, 0, k_all.shape[0], whole["q_rot"][:0], k_all, v_all, whole["o_loc"][:0],
                         d["gate"][:0], out[:0], err)
    assert p3.check_status(err) == 0 and torch.equal(out, before)


def test_forward_on_a_one_rank_nccl_group(p3):
    """zslab.forward as a rank calls it, through NCCL: one rank (every call here has one GPU),
    so no halo and a one-part all-gather; the result must be the whole-volume forward's."""
    import datetime
    import socket

    import torch.distributed as dist

    from geometry_aware_local_b200 import zslab
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda:0"))
    try:
        s = synth.Pack3DShape(Z=5, H=12, W=20, Hq=8, Hkv=2, rz=1, ry=3, rx=3, dtype="bf16", value_scale=0.125,
                              packing="random")
        inp = synth.make_inputs(s, seed=53)
        d = {k: v.cuda() for k, v in inp.items() if k != "sites"}
        cfg = p3.config_from_shape(s)
        out = zslab.forward(cfg, d, 0, 1)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    whole = whole_volume(p3, cfg, s, d)
    assert rel_err(out.float().cpu(), whole["out"].float().cpu()) <= 1e-2
    ref = oracle.forward(s, inp)["out"]
    assert rel_err(out.float().cpu().numpy(), ref) <= TOL["bf16"]
