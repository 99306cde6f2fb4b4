"""The z-slab split of one volume on one GPU: every rank's steps, in turn, in one process.

No rank waits on another here: every rank's zslab.Plan runs its phases in
turn (the boundary rows gathered by pack3d_gather_rows, summaries, RoPE and
local attention, the summary compaction, the query x summary stage), and the
two NCCL steps are replaced by copies between the plans' buffers.  Each rank
works on its extended lattice, whose origin is the true z of its first plane; the concatenation of all ranks' outputs must match the
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
    """Every rank's zslab.Plan phases on this GPU, the NCCL steps replaced by copies between the
    plans' buffers; returns the whole-volume arrays assembled from the ranks."""
    from geometry_aware_local_b200 import zslab
    plans, takes = [], []
    for r in range(world):
        idx, own = zslab.take_slab(d, zslab.make_plan(cfg, r, world))
        plan = zslab.Plan(cfg, own["coords"], r, world)
        for k, v in plan.inputs().items():
            v.copy_(own[k])
        plans.append(plan)
        takes.append(idx)
    for plan in plans:
        plan.pack_halo()
    for r, plan in enumerate(plans):
        below, above = plan.halo_views()
        if below is not None:                      # the rank below sent its last planes
            _, ks, vs = plans[r - 1].send["above"]
            below[0].copy_(ks)
            below[1].copy_(vs)
        if above is not None:                      # the rank above sent its first planes
            _, ks, vs = plans[r + 1].send["below"]
            above[0].copy_(ks)
            above[1].copy_(vs)
    for plan in plans:
        plan.local()
    parts = [plan.summary_part() for plan in plans]
    for plan in plans:                             # the all-gather, then the compaction
        if plan.uneven:
            plan.k_pad.copy_(torch.cat([k for k, _ in parts]))
            plan.v_pad.copy_(torch.cat([v for _, v in parts]))
            p3.gather_rows(plan.compact, plan.k_pad, plan.k_all)
            p3.gather_rows(plan.compact, plan.v_pad, plan.v_all)
        else:
            plan.k_all.copy_(torch.cat([k for k, _ in parts]))
            plan.v_all.copy_(torch.cat([v for _, v in parts]))
    res = dict(k_sum=plans[0].k_all, v_sum=plans[0].v_all, q_rot=torch.empty_like(d["q"]),
               out=torch.empty_like(d["q"]), o_loc=torch.empty(s.N, s.Hq, s.d_h, dtype=torch.float32, device="cuda"))
    for plan, idx in zip(plans, takes):
        t = plan.p.tokens
        res["out"][idx] = plan.attend()
        res["q_rot"][idx] = plan.q_rot[:t]
        res["o_loc"][idx] = plan.o_loc[:t]
        assert p3.check_status(plan.err) == 0
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


def test_single_rank_plan_needs_no_process_group(p3):
    """A one-rank Plan runs without torch.distributed (no exchange, the summaries are the volume's)."""
    from geometry_aware_local_b200 import zslab
    s = synth.Pack3DShape(Z=3, H=12, W=20, Hq=8, Hkv=2, dtype="bf16", value_scale=0.125, packing="random")
    inp = synth.make_inputs(s, seed=54)
    d = {k: v.cuda() for k, v in inp.items() if k != "sites"}
    cfg = p3.config_from_shape(s)
    plan = zslab.Plan(cfg, d["coords"], 0, 1)
    for k, v in plan.inputs().items():
        v.copy_(d[k])
    out = plan.forward()
    whole = whole_volume(p3, cfg, s, d)
    assert torch.equal(out, whole["out"])


@pytest.mark.parametrize("raw", [False, True])
def test_single_rank_plan_on_a_side_stream(p3, raw):
    """A Plan given its own stream (a torch stream, or the raw handle) runs every phase there, and
    its exchanges would run with that stream as torch's current one (the stream NCCL orders after)."""
    from geometry_aware_local_b200 import zslab
    s = synth.Pack3DShape(Z=4, H=12, W=20, Hq=8, Hkv=2, dtype="bf16", value_scale=0.125, packing="morton")
    inp = synth.make_inputs(s, seed=55)
    d = {k: v.cuda() for k, v in inp.items() if k != "sites"}
    cfg = p3.config_from_shape(s)
    side = torch.cuda.Stream()
    plan = zslab.Plan(cfg, d["coords"], 0, 1, stream=side.cuda_stream if raw else side)
    with plan._on_stream():
        assert torch.cuda.current_stream().cuda_stream == side.cuda_stream
    for k, v in plan.inputs().items():
        v.copy_(d[k])
    side.wait_stream(torch.cuda.current_stream())
    out = plan.forward()
    torch.cuda.current_stream().wait_stream(side)
    whole = whole_volume(p3, cfg, s, d)
    assert torch.equal(out, whole["out"])


@pytest.mark.parametrize("n,row_shape,dtype", [(1, (2, 64), torch.bfloat16), (1000, (2, 64), torch.bfloat16),
                                               (777, (8, 64), torch.float32), (5, (4,), torch.float32)])
def test_gather_rows_bit_exact(p3, n, row_shape, dtype):
    """pack3d_gather_rows: dst row i is src row idx[i], a negative index a zero row (byte moves only)."""
    gen = torch.Generator(device="cuda").manual_seed(n)
    src = torch.randn((3000,) + row_shape, generator=gen, device="cuda").to(dtype)
    idx = torch.randint(-1, 3000, (n,), generator=gen, device="cuda", dtype=torch.int32)
    dst = torch.full((n,) + row_shape, 7.0, device="cuda", dtype=dtype)
    p3.gather_rows(idx, src, dst)
    torch.cuda.synchronize()
    want = src.index_select(0, idx.clamp(min=0).long())
    want[idx < 0] = 0
    assert torch.equal(dst, want)
