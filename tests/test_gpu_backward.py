"""GPU parity of the training block (pack3d_forward_backward) against the float64 oracle.

Every gradient of L = <dOut, out> (dq, dk_loc, dv_loc, dk_cmp, dv_cmp, dscores,
dgate) and the forward output are compared element by element with the oracle's
chain-rule backward on the same seeded inputs (bf16 values widened exactly).
Tolerance: max |gpu - oracle| <= 1e-4 * max |oracle| (float) or 2e-2 * max |oracle|
(bf16), per tensor.  At 65k tokens the query-side gradients are compared on every
row and the key- and summary-side ones on seeded samples of keys and blocks.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
GRADS = ("dq", "dk_loc", "dv_loc", "dk_cmp", "dv_cmp", "dscores", "dgate")


@pytest.fixture(scope="module")
def p3(cuda_device):
    import geometry_aware_local_b200 as p3
    return p3


def rel_err(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(gpu - ref).max() / max(np.abs(ref).max(), 1e-30))


def run_fwd_bwd(p3, s, inp, dout, flags=0):
    cfg = p3.config_from_shape(s, flags)
    d = {k: v.cuda() for k, v in inp.items() if k != "sites"}
    do = dout.cuda()
    out = torch.empty_like(d["q"])
    grads = p3.empty_grads(d["q"], d["k_loc"], d["scores"], d["gate"])
    ws = torch.empty(p3.train_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    p3.forward_backward(cfg, d["coords"], d["q"], d["k_loc"], d["v_loc"], d["k_cmp"], d["v_cmp"], d["scores"],
                        d["gate"], do, out, grads, ws, err)
    assert p3.check_status(err) == 0
    res = {k: v.cpu() for k, v in grads.items()}
    res["out"] = out.cpu()
    return res


def small(**kw):
    base = dict(Z=3, H=12, W=20, Hq=8, Hkv=2, rz=1, ry=3, rx=3, dtype="bf16", value_scale=0.125)
    base.update(kw)
    return synth.Pack3DShape(**base)


CASES = [
    ("tiny-f32", synth.CONFIGS["tiny"], "raster", 0),
    ("tiny-f32-random", synth.CONFIGS["tiny"], "random", 0),
    ("ragged-bf16", small(), "random", 0),                       # tcgen05 forward paths, ragged bricks
    ("ragged-f32", small(dtype="f32", value_scale=1.0), "morton", 0),
    ("m-multi-bf16", small(Z=4, H=32, W=40), "random", 0),        # M = 320: several summary tiles + a tail
    ("g1-bf16", small(Hq=2, Hkv=2), "block", 0),
    ("g2-f32", small(Hq=4, Hkv=2, Z=2, H=8, W=8, dtype="f32", value_scale=1.0), "raster", 0),
    ("g8-bf16", small(Hq=8, Hkv=1), "random", 0),
    ("blocks222-bf16", small(Z=4, H=12, W=16, bz=2, by=2, bx=2), "block_morton", 0),
    ("window-2x1-bf16", small(Z=5, H=12, W=12, ry=2, rx=1), "morton", 0),
    ("simt-forward-bf16", small(), "random", 0x3),                # CUDA-core forward kernels on bf16
    ("coords-scaled-f32", small(dtype="f32", value_scale=1.0, coord_scale=(2.5, 0.5, 1.0)), "random", 0),
    ("z-light-bf16", small(m_z=6, m_y=13, m_x=13), "block", 0),
    # degenerate volumes with M >= 2 and blocks of >= 2 members (with one summary,
    # or one member per block, dk~ and dscores are zero by the softmax's invariance
    # and a tolerance relative to them is meaningless): two blocks whose window
    # covers nearly the whole volume, a one-row line, a column of 4x4 planes
    ("two-blocks-bf16", small(Z=1, H=4, W=8), "block", 0),
    ("two-blocks-f32", small(Z=1, H=4, W=8, dtype="f32", value_scale=1.0), "raster", 0),
    ("line-1x1x64-bf16", small(Z=1, H=1, W=64, by=1, bx=4), "morton", 0),
    ("z-column-bf16", small(Z=16, H=4, W=4), "random", 0),
]


@pytest.mark.parametrize("name,s,packing,flags", CASES, ids=[c[0] for c in CASES])
def test_forward_backward_matches_oracle(p3, name, s, packing, flags):
    inp = synth.make_inputs(s, packing, seed=4)
    dout = synth.make_dout(s, packing, seed=4)
    gpu = run_fwd_bwd(p3, s, inp, dout, flags)
    ref = oracle.backward(s, inp, dout)
    tol = TOL[s.dtype]
    for key in GRADS + ("out",):
        e = rel_err(gpu[key].double().numpy(), ref[key])
        assert e <= tol, f"{name}: {key} rel err {e:.3e} > {tol}"


TWO_TILE_CASES = [c for c in CASES if c[1].dtype == "bf16" and not c[3]]


@pytest.mark.parametrize("name,s,packing,flags", TWO_TILE_CASES, ids=[c[0] for c in TWO_TILE_CASES])
def test_two_tile_training_forward_matches_oracle(p3, name, s, packing, flags):
    """The training instantiation of the two-tile query x summary build (statistics and dgate in its
    epilogue), forced at small M, through every bf16 case: all gradients against the oracle."""
    inp = synth.make_inputs(s, packing, seed=4)
    dout = synth.make_dout(s, packing, seed=4)
    gpu = run_fwd_bwd(p3, s, inp, dout, flags | p3.FLAG_SUMMARY_TWO_TILE)
    ref = oracle.backward(s, inp, dout)
    for key in GRADS + ("out",):
        e = rel_err(gpu[key].double().numpy(), ref[key])
        assert e <= TOL["bf16"], f"{name}: {key} rel err {e:.3e}"


@pytest.mark.parametrize("build", ["two-tile", "one-tile"])
def test_forward_backward_large_m_sharp(p3, build):
    """28,672 tokens in 1x2x2 blocks, so M = 7,168 (56 tiles of 128 summaries), each query x summary
    build forced, with Q x 8 and K_loc / 8 (exact in bf16) making the summary softmax sharp.  Every
    gradient against the oracle's chain rule: dq, dgate and out on every row, the local key gradients on
    sampled keys, the summary-side ones on sampled blocks."""
    s = small(Z=4, H=64, W=112, by=2, bx=2, value_scale=1.0)
    inp = synth.make_inputs(s, "morton", seed=17)
    inp["q"] = (inp["q"].float() * 8.0).bfloat16()
    inp["k_loc"] = (inp["k_loc"].float() * 0.125).bfloat16()
    dout = synth.make_dout(s, "morton", seed=17)
    flags = p3.FLAG_SUMMARY_TWO_TILE if build == "two-tile" else p3.FLAG_SUMMARY_ONE_TILE
    gpu = run_fwd_bwd(p3, s, inp, dout, flags)
    rng = np.random.default_rng(23)
    keys = np.unique(np.concatenate([[0, s.N - 1], rng.choice(s.N, 254, replace=False)]))
    blocks = np.unique(np.concatenate([[0, s.M - 1], rng.choice(s.M, 62, replace=False)]))
    ref = oracle.backward(s, inp, dout, keys=keys, blocks=blocks)
    kt, tok = torch.from_numpy(keys), torch.from_numpy(ref["cmp_tokens"])
    checks = {"dq": (gpu["dq"], ref["dq"]), "dgate": (gpu["dgate"], ref["dgate"]), "out": (gpu["out"], ref["out"]),
              "dk_loc": (gpu["dk_loc"].index_select(0, kt), ref["dk_loc"]),
              "dv_loc": (gpu["dv_loc"].index_select(0, kt), ref["dv_loc"])}
    for k in ("dk_cmp", "dv_cmp", "dscores"):
        checks[k] = (gpu[k].index_select(0, tok), ref[k])
    for k, (a, b) in checks.items():
        e = rel_err(a.double().numpy(), b)
        assert e <= TOL["bf16"], f"{k} rel err {e:.3e}"


CENTER_CASES = [
    ("center-bf16", small(), "random", 0),
    ("center-f32", small(dtype="f32", value_scale=1.0), "morton", 0),
    ("center-blocks222-bf16", small(Z=4, H=12, W=16, bz=2, by=2, bx=2), "block", 0),
]


@pytest.mark.parametrize("name,s,packing,flags", CENTER_CASES, ids=[c[0] for c in CENTER_CASES])
def test_summary_center_forward_backward_matches_oracle(p3, name, s, packing, flags):
    """The summary-centre variant through the training block against the oracle's centre backward."""
    inp = synth.make_inputs(s, packing, seed=4)
    dout = synth.make_dout(s, packing, seed=4)
    gpu = run_fwd_bwd(p3, s, inp, dout, flags | p3.FLAG_SUMMARY_CENTER)
    ref = oracle.backward(s, inp, dout, center=True)
    tol = TOL[s.dtype]
    for key in GRADS + ("out",):
        e = rel_err(gpu[key].double().numpy(), ref[key])
        assert e <= tol, f"{name}: {key} rel err {e:.3e} > {tol}"


@pytest.mark.parametrize("flags", [0, 0x3])
def test_training_forward_output_equals_forward(p3, flags):
    """The training forward (statistics saved in the epilogue) leaves `out` bit for bit as pack3d_forward."""
    s = small(Z=4, H=32, W=40)
    inp = synth.make_inputs(s, "morton", seed=2)
    dout = synth.make_dout(s, "morton", seed=2)
    gpu = run_fwd_bwd(p3, s, inp, dout, flags)
    cfg = p3.config_from_shape(s, flags)
    d = {k: v.cuda() for k, v in inp.items() if k != "sites"}
    op = p3.Pack3D(cfg, "cuda")
    out = op(d["coords"], d["q"], d["k_loc"], d["v_loc"], d["k_cmp"], d["v_cmp"], d["scores"], d["gate"])
    op.check()
    assert torch.equal(out.cpu(), gpu["out"])


def test_gate_pinned_local_gives_zero_compressed_gradients(p3):
    s = small()
    inp = synth.make_inputs(s, "random", seed=6)
    inp["gate"][..., 0] = 40.0
    inp["gate"][..., 1] = -40.0
    gpu = run_fwd_bwd(p3, s, inp, synth.make_dout(s, "random", seed=6))
    for k in ("dk_cmp", "dv_cmp", "dscores"):
        assert gpu[k].abs().max().item() < 1e-20
    assert gpu["dk_loc"].abs().max().item() > 1e-4


def test_backward_is_deterministic_where_no_atomics(p3):
    """dq, dgate and out are written without atomics: identical across calls.  The key-side
    gradients are summed with float atomics and may differ in their last bits."""
    s = small(Z=4, H=32, W=40)
    inp = synth.make_inputs(s, "random", seed=8)
    dout = synth.make_dout(s, "random", seed=8)
    a = run_fwd_bwd(p3, s, inp, dout)
    b = run_fwd_bwd(p3, s, inp, dout)
    for k in ("dq", "dgate", "out"):
        assert torch.equal(a[k], b[k]), k
    # a different float summation order can move a bf16 result by one unit in the last place,
    # at most 2^-7 of its magnitude
    for k in ("dk_loc", "dv_loc", "dk_cmp", "dv_cmp", "dscores"):
        assert rel_err(a[k].double().numpy(), b[k].double().numpy()) <= 2.0 ** -7, k


def test_gradients_permute_with_the_packing(p3):
    """Proposition 1 carried through the chain rule: repacking permutes every gradient."""
    s = small(Z=4, H=16, W=24)
    base = run_fwd_bwd(p3, s, synth.make_inputs(s, "raster", seed=9), synth.make_dout(s, "raster", seed=9))
    for packing in ("morton", "random"):
        sites = torch.from_numpy(synth.packing_sites(s.Z, s.H, s.W, packing, 9, (s.bz, s.by, s.bx)))
        g = run_fwd_bwd(p3, s, synth.make_inputs(s, packing, seed=9), synth.make_dout(s, packing, seed=9))
        for k in GRADS:
            ref = base[k].index_select(0, sites).double().numpy()
            assert rel_err(g[k].double().numpy(), ref) <= 2e-2, (packing, k)


def test_forward_backward_65k_sampled(p3):
    """The 65k volume in the bench's configuration: query-side gradients on every row, key and
    summary gradients on seeded samples (the oracle's summary-side pass runs per sampled block)."""
    s = synth.CONFIGS["65k"]
    inp = synth.make_inputs(s, "morton", seed=0)
    dout = synth.make_dout(s, "morton", seed=0)
    gpu = run_fwd_bwd(p3, s, inp, dout)
    rng = np.random.default_rng(21)
    keys = np.unique(np.concatenate([[0, s.N - 1], rng.choice(s.N, 254, replace=False)]))
    blocks = np.unique(np.concatenate([[0, s.M - 1], rng.choice(s.M, 30, replace=False)]))
    ref = oracle.backward(s, inp, dout, keys=keys, blocks=blocks)
    tol = TOL["bf16"]
    kt = torch.from_numpy(keys)
    checks = {"dq": (gpu["dq"], ref["dq"]), "dgate": (gpu["dgate"], ref["dgate"]), "out": (gpu["out"], ref["out"]),
              "dk_loc": (gpu["dk_loc"].index_select(0, kt), ref["dk_loc"]),
              "dv_loc": (gpu["dv_loc"].index_select(0, kt), ref["dv_loc"])}
    tok = torch.from_numpy(ref["cmp_tokens"])
    for k in ("dk_cmp", "dv_cmp", "dscores"):
        checks[k] = (gpu[k].index_select(0, tok), ref[k])
    for k, (a, b) in checks.items():
        e = rel_err(a.double().numpy(), b)
        assert e <= tol, f"65k: {k} rel err {e:.3e} > {tol}"


def test_autograd_op_matches_forward_backward(p3):
    """geometry_aware_local_b200.attention: torch.autograd gradients equal pack3d_forward_backward's,
    and the forward output equals pack3d_forward's; the gradients match the oracle."""
    s = small(Z=4, H=16, W=24)
    inp = synth.make_inputs(s, "random", seed=12)
    dout = synth.make_dout(s, "random", seed=12)
    cfg = p3.config_from_shape(s)
    names = ("q", "k_loc", "v_loc", "k_cmp", "v_cmp", "scores", "gate")
    d = {k: inp[k].cuda().requires_grad_(k in names) for k in ("coords",) + names}
    out = p3.attention(cfg, d["coords"], *[d[k] for k in names])
    out.backward(dout.cuda())
    ref = run_fwd_bwd(p3, s, inp, dout)
    assert torch.equal(out.detach().cpu(), ref["out"])
    grad_of = dict(zip(names, ("dq", "dk_loc", "dv_loc", "dk_cmp", "dv_cmp", "dscores", "dgate")))
    oref = oracle.backward(s, inp, dout)
    for k, gname in grad_of.items():
        g = d[k].grad.cpu()
        assert rel_err(g.double().numpy(), ref[gname].double().numpy()) <= 2.0 ** -7, k
        assert rel_err(g.double().numpy(), oref[gname]) <= TOL["bf16"], k
