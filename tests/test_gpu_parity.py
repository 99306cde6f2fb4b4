"""GPU parity: every stage of the CUDA path against the float64 oracle.

The CUDA path is called through the C ABI (ctypes binding); the oracle is the
plain definition of each stage.  Both see the same seeded inputs (bf16 values
widened exactly for the oracle).  Tolerances follow the operator's contract:
max |gpu - oracle| <= 1e-4 * max |oracle| on float inputs and
<= 2e-2 * max |oracle| on bf16 inputs with float accumulation; the index map and
block membership are compared bit for bit.
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


def to_dev(inp):
    return {k: (v.cuda() if k != "sites" else v) for k, v in inp.items()}


def rel_err(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(gpu - ref).max() / max(np.abs(ref).max(), 1e-30))


def run_stages(p3, s, d, flags=0):
    """Every entry point in order; returns the intermediates as CPU tensors."""
    cfg = p3.config_from_shape(s, flags)
    dt = d["q"].dtype
    dev = d["q"].device
    err = torch.zeros(4, dtype=torch.int32, device=dev)
    g2p = torch.empty(s.N, dtype=torch.int32, device=dev)
    mem = torch.empty(s.M, s.v, dtype=torch.int32, device=dev)
    p3.build_index(cfg, d["coords"], g2p, mem, err)
    qr = torch.empty_like(d["q"])
    kr = torch.empty_like(d["k_loc"])
    p3.rope(cfg, d["coords"], d["q"], qr, s.Hq)
    p3.rope(cfg, d["coords"], d["k_loc"], kr, s.Hkv)
    ks = torch.empty(s.M, s.Hkv, s.d_h, dtype=dt, device=dev)
    vs = torch.empty_like(ks)
    p3.build_summaries(cfg, mem, d["k_cmp"], d["v_cmp"], d["scores"], ks, vs)
    ol = torch.empty(s.N, s.Hq, s.d_h, dtype=torch.float32, device=dev)
    p3.local_attn(cfg, g2p, qr, kr, d["v_loc"], ol, err)
    oc = torch.empty_like(d["q"])
    p3.summary_attn(cfg, qr, ks, vs, None, None, oc, err)
    out = torch.empty_like(d["q"])
    p3.summary_attn(cfg, qr, ks, vs, ol, d["gate"], out, err)
    assert p3.check_status(err) == 0
    return {k: v.cpu() for k, v in dict(g2p=g2p, members=mem, q_rot=qr, k_rot=kr, k_sum=ks, v_sum=vs,
                                         o_loc=ol, o_cmp=oc, out=out).items()}


def run_forward(p3, s, d, flags=0):
    cfg = p3.config_from_shape(s, flags)
    op = p3.Pack3D(cfg, d["q"].device)
    out = op(d["coords"], d["q"], d["k_loc"], d["v_loc"], d["k_cmp"], d["v_cmp"], d["scores"], d["gate"])
    op.check()
    return out.cpu()


def small(**kw):
    base = dict(Z=3, H=12, W=20, Hq=8, Hkv=2, rz=1, ry=3, rx=3, dtype="bf16", value_scale=0.125)
    base.update(kw)
    return synth.Pack3DShape(**base)


# ------------------------------------------------------------ stage by stage -----

STAGE_CASES = [
    ("tiny", synth.CONFIGS["tiny"], "raster"),
    ("tiny-f32-random", synth.CONFIGS["tiny"].replace(packing="random"), "random"),
    ("ragged-bf16", small(), "random"),                      # W, H not multiples of the 8x8 brick
    ("ragged-f32", small(dtype="f32", value_scale=1.0), "morton"),
    ("g1", small(Hq=2, Hkv=2), "block"),
    ("g2", small(Hq=4, Hkv=2, Z=2, H=8, W=8), "raster"),
    ("g8", small(Hq=8, Hkv=1), "random"),
    ("m-tail", small(Z=2, H=20, W=24), "morton"),              # M = 60: a partial summary tile
    ("m-multi", small(Z=4, H=32, W=40), "random"),             # M = 320: several tiles + tail
    ("ragged-brick", small(Z=3, H=10, W=14, by=2, bx=2), "random"),  # 2x4x4 bricks cut in z, y and x
    ("window-2x1", small(Z=5, H=12, W=12, ry=2, rx=1), "morton"),     # 8x6 halo planes (48 keys)
    ("window-1x1x1", small(Z=4, H=8, W=8, ry=1, rx=1, rz=1), "block"),
    # summaries at Hkv = 4 and 8: two and four chunk slots per lane (bf16 / float)
    ("hkv4", small(Hq=8, Hkv=4), "random"),
    ("hkv8-f32", small(Hq=8, Hkv=8, dtype="f32", value_scale=1.0), "block"),
    ("hkv4-f32", small(Hq=8, Hkv=4, dtype="f32", value_scale=1.0), "morton"),
    # rotary configuration knobs: normalised coordinates, z rescaled, z-light and z-heavy pair splits
    ("coords-normalised", small(Z=4, H=16, W=24, coord_scale=(1 / 3, 1 / 15, 1 / 23)), "block_morton"),
    ("z-rescaled-f32", small(dtype="f32", value_scale=1.0, coord_scale=(2.5, 1.0, 1.0)), "random"),
    ("z-light", small(m_z=6, m_y=13, m_x=13), "block_morton"),
    ("z-heavy", small(m_z=16, m_y=8, m_x=8), "random"),
    # degenerate volumes: one block (M = 1, so every query's summary softmax has a
    # single term, and the 3x7x7 window covers the whole 1x4x4 volume), one token,
    # a one-row line (the y window clipped to a single row), a column of 4x4 planes
    ("one-block-bf16", small(Z=1, H=4, W=4), "random"),
    ("one-block-f32", small(Z=1, H=4, W=4, dtype="f32", value_scale=1.0), "raster"),
    ("one-token", small(Z=1, H=1, W=1, bz=1, by=1, bx=1), "raster"),
    ("line-1x1x64", small(Z=1, H=1, W=64, by=1, bx=4), "morton"),
    ("z-column", small(Z=16, H=4, W=4), "random"),
]


@pytest.mark.parametrize("name,s,packing", STAGE_CASES, ids=[c[0] for c in STAGE_CASES])
def test_stages_match_oracle(p3, name, s, packing):
    inp = synth.make_inputs(s, packing, seed=3)
    gpu = run_stages(p3, s, to_dev(inp))
    ref = oracle.forward(s, inp)
    tol = TOL[s.dtype]
    assert np.array_equal(gpu["g2p"].numpy(), ref["g2p"])
    assert np.array_equal(gpu["members"].numpy(), ref["members"])
    for key in ("q_rot", "k_rot", "k_sum", "v_sum", "o_loc", "o_cmp", "out"):
        e = rel_err(gpu[key].double().numpy(), ref[key])
        assert e <= tol, f"{name}: {key} rel err {e:.3e} > {tol}"


BF16_STAGE_CASES = [c for c in STAGE_CASES if c[1].dtype == "bf16"]


@pytest.mark.parametrize("name,s,packing", BF16_STAGE_CASES, ids=[c[0] for c in BF16_STAGE_CASES])
def test_two_tile_build_matches_oracle(p3, name, s, packing):
    """The two-tile query x summary build (one CTA per SM, chosen by size only above 48 summary
    tiles) forced on every bf16 stage case: its compressed branch and gate against the oracle."""
    inp = synth.make_inputs(s, packing, seed=3)
    gpu = run_stages(p3, s, to_dev(inp), flags=p3.FLAG_SUMMARY_TWO_TILE)
    ref = oracle.forward(s, inp)
    for key in ("o_cmp", "out"):
        e = rel_err(gpu[key].double().numpy(), ref[key])
        assert e <= TOL["bf16"], f"{name}: {key} rel err {e:.3e}"


@pytest.mark.parametrize("s", [small(Z=4, H=32, W=40), small(Z=3, H=10, W=14, by=2, bx=2), small(Hq=8, Hkv=1)],
                         ids=["m-multi", "ragged-brick", "g8"])
def test_one_and_two_tile_builds_agree(p3, s):
    """The one-tile build walks the summaries in tiles of 96, the two-tile build in tiles of 128: the
    same products in the same order, with the row sums grouped differently, so o_cmp, the gated
    output and the training forward's output and gradients agree to float rounding (within two bf16
    ulps of the largest value); each build is checked against the oracle elsewhere."""
    d = to_dev(synth.make_inputs(s, "random", seed=14))
    a = run_stages(p3, s, d, flags=p3.FLAG_SUMMARY_ONE_TILE)
    b = run_stages(p3, s, d, flags=p3.FLAG_SUMMARY_TWO_TILE)
    for k in ("o_cmp", "out"):
        assert rel_err(a[k].float().numpy(), b[k].float().numpy()) <= 8e-3, k
    dout = synth.make_dout(s, "random", seed=14).cuda()
    res = []
    for flags in (p3.FLAG_SUMMARY_ONE_TILE, p3.FLAG_SUMMARY_TWO_TILE):
        cfg = p3.config_from_shape(s, flags)
        out = torch.empty_like(d["q"])
        grads = p3.empty_grads(d["q"], d["k_loc"], d["scores"], d["gate"])
        ws = torch.empty(p3.train_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
        err = torch.zeros(4, dtype=torch.int32, device="cuda")
        p3.forward_backward(cfg, d["coords"], d["q"], d["k_loc"], d["v_loc"], d["k_cmp"], d["v_cmp"], d["scores"],
                            d["gate"], dout, out, grads, ws, err)
        assert p3.check_status(err) == 0
        res.append((out.float().cpu(), grads["dgate"].float().cpu(), grads["dq"].float().cpu()))
    for i, k in enumerate(("out", "dgate", "dq")):
        assert rel_err(res[0][i].numpy(), res[1][i].numpy()) <= 8e-3, k


def sharp_inputs(s, packing, seed):
    """Inputs whose summary softmax is sharp: Q x 8 and K_loc / 8 (exact in bf16) on top of value_scale 1,
    so the compressed logits have a standard deviation of about 3 (a few summaries carry each row) while
    the local logits stay about N(0,1).  A wrong summary tile, ring stage or rescale then moves o_cmp by
    the size of a summary value instead of by a fraction of a flat average."""
    inp = synth.make_inputs(s, packing, seed=seed)
    inp["q"] = (inp["q"].float() * 8.0).to(inp["q"].dtype)
    inp["k_loc"] = (inp["k_loc"].float() * 0.125).to(inp["k_loc"].dtype)
    return inp


@pytest.mark.parametrize("build", ["two-tile", "one-tile"])
def test_large_m_sharp_logits(p3, build):
    """131,072 tokens, M = 8,192 (64 tiles of 128 summaries, 86 of 96) with a sharp summary softmax,
    each build forced: o_cmp and out on every row of the first, a middle and the last two-tile CTA's
    query tiles (two 128-row tiles per kv head each) and on 1,024 sampled tokens, element by element."""
    s = synth.Pack3DShape(Z=8, H=64, W=256, Hq=8, Hkv=2, value_scale=1.0)
    inp = sharp_inputs(s, "random", seed=7)
    flags = p3.FLAG_SUMMARY_TWO_TILE if build == "two-tile" else p3.FLAG_SUMMARY_ONE_TILE
    gpu = run_stages(p3, s, to_dev(inp), flags=flags)
    per_cta = 2 * 128 // (s.Hq // s.Hkv)        # tokens of one two-tile CTA (both kv heads run it)
    mid = (s.N // 2) // per_cta * per_cta
    full_tiles = np.concatenate([np.arange(0, per_cta), np.arange(mid, mid + per_cta),
                                 np.arange(s.N - per_cta, s.N)])
    rows = np.unique(np.concatenate([full_tiles, synth.sample_rows(s.N, 1024, seed=5)]))
    ref = oracle.forward(s, inp, rows)
    # the softmax really is sharp: a few dozen of the 8,192 summaries carry each row
    logits = np.einsum("rd,md->rm", ref["q_rot"][:64, 0], ref["k_sum"][:, 0]) * s.softmax_scale
    pr = np.exp(logits - logits.max(1, keepdims=True))
    pr /= pr.sum(1, keepdims=True)
    assert np.median(1.0 / (pr ** 2).sum(1)) < 64
    for key in ("o_cmp", "out"):
        e = rel_err(gpu[key][rows].double().numpy(), ref[key])
        assert e <= TOL["bf16"], f"{key} rel err {e:.3e}"


CENTER_CASES = [
    ("bf16-warp", small(), "random"),                                  # warp-per-block kernel
    ("f32-tiny", synth.CONFIGS["tiny"], "raster"),
    ("bf16-v4", small(Z=3, H=10, W=14, by=2, bx=2), "morton"),         # block volume 4
    ("bf16-v32", small(Z=4, H=8, W=8, bz=2), "block"),                 # block volume 32 (generic kernel)
]


@pytest.mark.parametrize("name,s,packing", CENTER_CASES, ids=[c[0] for c in CENTER_CASES])
def test_summary_center_variant_matches_oracle(p3, name, s, packing):
    """PACK3D_FLAG_SUMMARY_CENTER: summaries and the whole forward pass against the oracle's variant."""
    inp = synth.make_inputs(s, packing, seed=13)
    gpu = run_stages(p3, s, to_dev(inp), flags=p3.FLAG_SUMMARY_CENTER)
    ref = oracle.forward(s, inp, center=True)
    tol = TOL[s.dtype]
    for key in ("k_sum", "v_sum", "o_cmp", "out"):
        e = rel_err(gpu[key].double().numpy(), ref[key])
        assert e <= tol, f"{name}: {key} rel err {e:.3e} > {tol}"
    exact = oracle.forward(s, inp)
    assert rel_err(ref["k_sum"], exact["k_sum"]) > 2 * tol      # the variant differs from the exact form


def test_simt_and_tensor_core_summary_paths_agree(p3):
    s = small(Z=4, H=32, W=40)
    d = to_dev(synth.make_inputs(s, "random", seed=4))
    a = run_stages(p3, s, d)
    b = run_stages(p3, s, d, flags=p3.FLAG_SIMT_SUMMARY)
    assert rel_err(a["out"].double(), b["out"].double()) <= TOL["bf16"]


@pytest.mark.parametrize("shape", [small(Z=4, H=32, W=40), small(Z=3, H=10, W=14, by=2, bx=2)])
def test_simt_and_tensor_core_local_paths_agree(p3, shape):
    d = to_dev(synth.make_inputs(shape, "random", seed=6))
    a = run_stages(p3, shape, d)
    b = run_stages(p3, shape, d, flags=p3.FLAG_SIMT_LOCAL)
    assert rel_err(a["o_loc"].double(), b["o_loc"].double()) <= TOL["bf16"]


@pytest.mark.parametrize("order", ["rising", "falling"])
def test_summary_attention_extreme_logit_ranges(p3, order):
    # Logits that grow by far more than the float exponent range between
    # summary tiles (rising) force the kernel's recompute-and-rescale path;
    # falling logits underflow later tiles.  Both must still match the oracle.
    s = small(Z=4, H=32, W=32)          # N = 4096, M = 256 -> two 128-summary tiles
    gen = torch.Generator().manual_seed(11)
    q = torch.randn(s.N, s.Hq, 64, generator=gen)
    ks = torch.randn(s.M, s.Hkv, 64, generator=gen) * 0.05
    vs = torch.randn(s.M, s.Hkv, 64, generator=gen)
    big = slice(128, 256) if order == "rising" else slice(0, 128)
    ks[big] = q[:128].reshape(128, s.Hq, 64)[:, ::4][:, :s.Hkv] * 8.0   # aligned with some queries
    q, ks, vs = (t.bfloat16() for t in (q, ks, vs))
    cfg = p3.config_from_shape(s)
    out = torch.empty(s.N, s.Hq, 64, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    p3.summary_attn(cfg, q.cuda(), ks.cuda(), vs.cuda(), None, None, out, err)
    assert p3.check_status(err) == 0
    rows = synth.sample_rows(s.N, 300, seed=4)
    ref = oracle.summary_attn(s, q[torch.from_numpy(rows)], ks, vs)
    got = out.cpu()[torch.from_numpy(rows)].double().numpy()
    assert np.isfinite(got).all()
    assert rel_err(got, ref) <= TOL["bf16"]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_rope_qk_equals_two_rope_calls(p3, dtype):
    """The fused Q/K launch computes exactly what the single-tensor entry point does."""
    s = small(Z=4, H=16, W=24, dtype=dtype)
    d = to_dev(synth.make_inputs(s, "random", seed=11))
    cfg = p3.config_from_shape(s)
    qa, ka = torch.empty_like(d["q"]), torch.empty_like(d["k_loc"])
    p3.rope(cfg, d["coords"], d["q"], qa, s.Hq)
    p3.rope(cfg, d["coords"], d["k_loc"], ka, s.Hkv)
    qb, kb = torch.empty_like(qa), torch.empty_like(ka)
    p3.rope_qk(cfg, d["coords"], d["q"], qb, d["k_loc"], kb)
    torch.cuda.synchronize()
    assert torch.equal(qa, qb) and torch.equal(ka, kb)


@pytest.mark.parametrize("name", ["tiny", "small", "65k", "131k"])
def test_forward_host_equals_forward(p3, name):
    """The host-buffer pipeline (copies overlapped, summary stage in token chunks) gives exactly the
    device-buffer forward pass's output; 131k tokens (M = 8,192) chunks the two-tile build."""
    s = {"tiny": synth.CONFIGS["tiny"], "small": small(Z=4, H=16, W=24), "65k": synth.CONFIGS["65k"],
         "131k": synth.Pack3DShape(Z=8, H=64, W=256, Hq=8, Hkv=2, packing="block")}[name]
    inp = synth.make_inputs(s, s.packing, seed=5)
    d = to_dev(inp)
    ref = run_forward(p3, s, d)
    cfg = p3.config_from_shape(s)
    names = ("coords", "q", "k_loc", "v_loc", "k_cmp", "v_cmp", "scores", "gate")
    hin = {k: inp[k].contiguous().pin_memory() for k in names}
    hout = torch.empty(tuple(ref.shape), dtype=ref.dtype).pin_memory()
    ws = torch.empty(p3.host_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    pipe = p3.Pipeline()
    for _ in range(2):   # a second call reuses the pipeline and the staging area
        hout.zero_()
        p3.forward_host(pipe, cfg, *(hin[k] for k in names), hout, ws, err)
        assert p3.check_status(err) == 0
        assert torch.equal(hout, ref.cpu())
    pipe.close()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_empty_volume(p3, dtype):
    """N = 0 (a zero lattice extent): the forward op, the host-buffer pipeline and
    the differentiable op return empty outputs and empty gradients, status OK."""
    cfg = p3.make_config(0, 64, 64, dtype=dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    dev = "cuda"
    coords = torch.empty(0, 3, dtype=torch.int32, device=dev)
    q = torch.empty(0, 8, 64, dtype=tdt, device=dev)
    kv = [torch.empty(0, 2, 64, dtype=tdt, device=dev) for _ in range(4)]
    scores = torch.empty(0, 2, dtype=torch.float32, device=dev)
    gate = torch.empty(0, 8, 2, dtype=torch.float32, device=dev)
    op = p3.Pack3D(cfg, dev)
    out = op(coords, q, *kv, scores, gate)
    op.check()
    assert out.shape == (0, 8, 64)

    # (no copy is made for N = 0, so the host tensors need not be page-locked)
    hin = [t.cpu() for t in (coords, q, *kv, scores, gate)]
    hout = torch.empty(0, 8, 64, dtype=tdt)
    ws = torch.empty(p3.host_workspace_bytes(cfg), dtype=torch.uint8, device=dev)
    err = torch.zeros(4, dtype=torch.int32, device=dev)
    pipe = p3.Pipeline()
    p3.forward_host(pipe, cfg, *hin, hout, ws, err)
    pipe.close()
    assert p3.check_status(err) == 0

    leaves = [t.clone().requires_grad_(True) for t in (q, *kv, scores, gate)]
    y = p3.attention(cfg, coords, *leaves)
    y.float().sum().backward()
    for t in leaves:
        assert t.grad is not None and t.grad.shape == t.shape


@pytest.mark.parametrize("name", ["small", "65k"])
def test_forward_is_deterministic(p3, name):
    # Every kernel computes each output from a fixed sequence of operations, so
    # repeated runs on the same inputs must agree bit for bit (a race or a read
    # of uninitialised state shows up here first).
    s = synth.CONFIGS["65k"] if name == "65k" else small(Z=4, H=16, W=24)
    d = to_dev(synth.make_inputs(s, s.packing, seed=8))
    outs = [run_forward(p3, s, d) for _ in range(3)]
    assert all(torch.equal(outs[0], o) for o in outs[1:])


# ------------------------------------------------------------ index map ---------

@pytest.mark.parametrize("packing", synth.PACKINGS)
def test_index_map_bit_exact_65k(p3, packing):
    s = synth.CONFIGS["65k"]
    coords = torch.from_numpy(synth.coords_for(s, packing))
    cfg = p3.config_from_shape(s)
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    g2p = torch.empty(s.N, dtype=torch.int32, device="cuda")
    mem = torch.empty(s.M, s.v, dtype=torch.int32, device="cuda")
    p3.build_index(cfg, coords.cuda(), g2p, mem, err)
    assert p3.check_status(err) == 0
    st, rg, rm = oracle.build_index(s, coords)
    assert st == 0
    assert np.array_equal(g2p.cpu().numpy(), rg) and np.array_equal(mem.cpu().numpy(), rm)


def test_bad_coordinates_are_reported(p3):
    s = small()
    cfg = p3.config_from_shape(s)
    coords = torch.from_numpy(synth.coords_for(s, "random")).clone()
    coords[7] = coords[11]
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    g2p = torch.empty(s.N, dtype=torch.int32, device="cuda")
    mem = torch.empty(s.M, s.v, dtype=torch.int32, device="cuda")
    p3.build_index(cfg, coords.cuda(), g2p, mem, err)
    assert p3.check_status(err) == 5
    coords = torch.from_numpy(synth.coords_for(s, "raster")).clone()
    coords[3, 2] = s.W
    p3.build_index(cfg, coords.cuda(), g2p, mem, err)
    assert p3.check_status(err) == 5
    assert p3.check_status(err) == 0   # the word was cleared


# ------------------------------------------------------------ whole forward -----

def test_forward_tiny_full(p3):
    s = synth.CONFIGS["tiny"]
    inp = synth.make_inputs(s, s.packing, seed=0)
    out = run_forward(p3, s, to_dev(inp))
    ref = oracle.forward(s, inp)["out"]
    assert rel_err(out.double().numpy(), ref) <= TOL["f32"]


def test_forward_65k_sampled_rows(p3):
    s = synth.CONFIGS["65k"]
    inp = synth.make_inputs(s, s.packing, seed=0)
    out = run_forward(p3, s, to_dev(inp))
    rows = synth.sample_rows(s.N, 1024, seed=1)
    ref = oracle.forward(s, inp, rows)["out"]
    assert rel_err(out[rows].double().numpy(), ref) <= TOL["bf16"]


def test_stress_packing_equivariance_65k(p3):
    # Proposition 1: out under packing P equals P applied to the raster output.
    s = synth.CONFIGS["stress"]
    sv = synth.draw_site_values(s, 5)
    base = synth.make_inputs(s, "raster", 5, sv)
    ref = run_forward(p3, s, to_dev(base)).double()
    rows = synth.sample_rows(s.N, 256, seed=2)
    oref = oracle.forward(s, base, rows)["out"]
    assert rel_err(ref[rows].numpy(), oref) <= TOL["bf16"]
    for packing in ("morton", "block", "random", "block_morton"):
        inp = synth.make_inputs(s, packing, 5, sv)
        out = run_forward(p3, s, to_dev(inp)).double()
        sites = inp["sites"]
        assert rel_err(out.numpy(), ref[sites].numpy()) <= TOL["bf16"], packing


@pytest.mark.parametrize("name", ["262k", "1m"])
def test_forward_large_sampled_rows(p3, name):
    s = synth.CONFIGS[name]
    inp = synth.make_inputs(s, s.packing, seed=0)
    out = run_forward(p3, s, to_dev(inp))
    rows = synth.sample_rows(s.N, 128, seed=3)
    ref = oracle.forward(s, inp, rows)["out"]
    assert rel_err(out[rows].double().numpy(), ref) <= TOL["bf16"]
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("name", ["4m", "8m"])
def test_forward_query_tiled_sizes_sampled_rows(p3, name):
    """4M and 8M tokens (M = 262,144 and 524,288 summaries): element offsets of q, out and
    o_loc pass 2^31 (4M x 8 heads x 64 = 2^31, 8M twice that), and the query x summary
    kernel walks 2,048 and 4,096 summary tiles.  Values are drawn on the device (the host
    recipe's float32 draws would not fit); the sampled rows include the first and the last
    32 packed rows, and the oracle gets the same values copied back."""
    s = synth.CONFIGS[name]
    d = synth.make_inputs_on_device(s, s.packing, seed=0)
    out = run_forward(p3, s, d)
    rows = np.unique(np.concatenate([synth.sample_rows(s.N, 96, seed=5), np.arange(s.N - 32, s.N)]))
    inp = {k: v.cpu() for k, v in d.items()}
    del d
    torch.cuda.empty_cache()
    ref = oracle.forward(s, inp, rows)
    assert rel_err(out[rows].double().numpy(), ref["out"]) <= TOL["bf16"]
    assert rel_err(out[-32:].double().numpy(), ref["out"][-32:]) <= TOL["bf16"]


def test_exp2_fma_against_reference(p3):
    """The FMA-pipe exponential of the one-tile query x summary build (pack3d_exp2_fma_eval) over the
    inputs the kernel feeds it (x <= 8 after the lazy maximum; masked columns at -inf): relative error
    within the fit's 7.5e-5 (plus float rounding) against a float64 2^x, and ~2.4e-38 for x <= -125."""
    x = torch.cat([torch.linspace(-125.0, 8.0, 2_000_001), torch.arange(-125, 9, dtype=torch.float32),
                   torch.arange(-125, 8, dtype=torch.float32) + 0.5,
                   torch.tensor([-0.5, 0.5, 1e-7, -1e-7, 0.0])]).cuda()
    y = torch.empty_like(x)
    p3.exp2_fma_eval(x, y)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref) / ref).abs().max().item()
    assert rel <= 8e-5, rel
    low = torch.tensor([-125.0, -126.0, -200.0, -1e30, float("-inf")], device="cuda")
    yl = torch.empty_like(low)
    p3.exp2_fma_eval(low, yl)
    assert (yl > 0).all() and (yl <= 2.4e-38).all() and torch.isfinite(yl).all()
