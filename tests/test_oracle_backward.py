"""Pins of the float64 oracle's backward pass (the training block's gradients).

The backward oracle applies the chain rule stage by stage; it is pinned here
against something other than itself:
* central finite differences of the (separately pinned) forward oracle:
  L(x) = <dOut, out(x)>, so <grad_x L, delta> must equal
  (L(x + eps delta) - L(x - eps delta)) / (2 eps) for random directions delta
  and for single elements of every input (a dropped term, a wrong sign, a
  transposed rotation or a swapped head map fails one of them);
* invariants of the softmaxes: the two gate gradients of a row sum to zero,
  and the score gradients of one block and kv head sum to zero (a softmax is
  unchanged by adding a constant to its logits);
* special cases: with the gate pinned to the local branch the compressed-side
  gradients vanish; under a repacking the gradients permute with the tokens
  (Proposition 1 of Key design 1 carried through the chain rule).
"""
import numpy as np
import pytest

import oracle
import synth

INPUTS = ("q", "k_loc", "v_loc", "k_cmp", "v_cmp", "scores", "gate")
GRAD = {"q": "dq", "k_loc": "dk_loc", "v_loc": "dv_loc", "k_cmp": "dk_cmp", "v_cmp": "dv_cmp",
        "scores": "dscores", "gate": "dgate"}

CASES = [
    ("tiny", synth.CONFIGS["tiny"], "random"),
    # two kv heads of two q heads each, 2x2x2 blocks, unequal radii, a short
    # rotary split and scaled coordinates
    ("g2-blocks222", synth.Pack3DShape(Z=4, H=6, W=8, Hq=4, Hkv=2, bz=2, by=2, bx=2, rz=1, ry=2, rx=1,
                                       m_z=4, m_y=6, m_x=5, dtype="f32", value_scale=1.0,
                                       coord_scale=(0.5, 1.0, 0.25)), "morton"),
]


def f64_inputs(s, packing, seed=5):
    inp = synth.make_inputs(s, packing, seed=seed)
    out = {"coords": inp["coords"].numpy().astype(np.int32)}
    for k in INPUTS:
        out[k] = inp[k].double().numpy().copy()
    return out


def loss(s, inp, dout):
    return float(np.sum(oracle.forward(s, inp)["out"] * dout))


@pytest.fixture(scope="module", params=CASES, ids=[c[0] for c in CASES])
def case(request):
    _, s, packing = request.param
    inp = f64_inputs(s, packing)
    dout = synth.make_dout(s, packing, seed=5).double().numpy()
    grads = oracle.backward(s, inp, dout)
    return s, inp, dout, grads


@pytest.mark.parametrize("name", INPUTS)
def test_directional_derivative_matches_finite_difference(case, name):
    s, inp, dout, grads = case
    rng = np.random.default_rng(11)
    delta = rng.standard_normal(inp[name].shape)
    eps = 1e-6
    plus = dict(inp, **{name: inp[name] + eps * delta})
    minus = dict(inp, **{name: inp[name] - eps * delta})
    fd = (loss(s, plus, dout) - loss(s, minus, dout)) / (2 * eps)
    an = float(np.sum(grads[GRAD[name]] * delta))
    assert abs(fd - an) <= 1e-6 * max(abs(an), 1e-3), f"{name}: fd {fd!r} vs analytic {an!r}"


@pytest.mark.parametrize("name", INPUTS)
def test_single_elements_match_finite_difference(case, name):
    s, inp, dout, grads = case
    rng = np.random.default_rng(17)
    g = grads[GRAD[name]]
    flat = rng.choice(g.size, size=4, replace=False)
    # include the largest-magnitude entry so at least one probe is well above rounding
    flat[0] = int(np.argmax(np.abs(g)))
    eps = 1e-6
    for f in flat:
        idx = np.unravel_index(f, g.shape)
        plus = {k: (v.copy() if k == name else v) for k, v in inp.items()}
        minus = {k: (v.copy() if k == name else v) for k, v in inp.items()}
        plus[name][idx] += eps
        minus[name][idx] -= eps
        fd = (loss(s, plus, dout) - loss(s, minus, dout)) / (2 * eps)
        scale = max(np.abs(g).max(), 1e-6)
        assert abs(fd - g[idx]) <= 1e-6 * scale, f"{name}{idx}: fd {fd!r} vs analytic {g[idx]!r}"


def test_gate_gradients_sum_to_zero(case):
    _, _, _, grads = case
    dg = grads["dgate"]
    assert np.abs(dg.sum(axis=-1)).max() <= 1e-12 * max(np.abs(dg).max(), 1.0)


def test_block_score_gradients_sum_to_zero(case):
    s, inp, _, grads = case
    _, _, mem = oracle.build_index(s, inp["coords"])
    ds = grads["dscores"]                       # [N, Hkv], packed order
    per_block = ds[mem.reshape(-1)].reshape(s.M, s.v, s.Hkv).sum(axis=1)
    assert np.abs(per_block).max() <= 1e-12 * max(np.abs(ds).max(), 1.0)


def test_gate_pinned_local_zeroes_compressed_gradients():
    s = CASES[1][1]
    inp = f64_inputs(s, "random")
    inp["gate"][..., 0] = 40.0
    inp["gate"][..., 1] = -40.0
    dout = synth.make_dout(s, "random", seed=5).double().numpy()
    g = oracle.backward(s, inp, dout)
    for k in ("dk_cmp", "dv_cmp", "dscores"):
        assert np.abs(g[k]).max() < 1e-30
    assert np.abs(g["dk_loc"]).max() > 1e-3 and np.abs(g["dv_loc"]).max() > 1e-3


def test_gradients_permute_with_the_packing():
    s = CASES[1][1]
    ref_inp = f64_inputs(s, "raster")
    ref = oracle.backward(s, ref_inp, synth.make_dout(s, "raster", seed=5).double().numpy())
    for packing in ("morton", "random"):
        inp = f64_inputs(s, packing)
        sites = synth.packing_sites(s.Z, s.H, s.W, packing, 5, (s.bz, s.by, s.bx))
        g = oracle.backward(s, inp, synth.make_dout(s, packing, seed=5).double().numpy())
        for k in ("dq", "dk_loc", "dv_loc", "dk_cmp", "dv_cmp", "dscores", "dgate"):
            np.testing.assert_allclose(g[k], ref[k][sites], rtol=0, atol=1e-12 * np.abs(ref[k]).max())


def test_sampled_keys_and_blocks_equal_the_full_backward():
    s, packing = CASES[1][1], "morton"
    inp = f64_inputs(s, packing)
    dout = synth.make_dout(s, packing, seed=5).double().numpy()
    full = oracle.backward(s, inp, dout)
    keys = np.array([0, 7, s.N - 1])
    blocks = np.array([1, s.M - 1])
    part = oracle.backward(s, inp, dout, keys=keys, blocks=blocks)
    np.testing.assert_array_equal(part["dk_loc"], full["dk_loc"][keys])
    np.testing.assert_array_equal(part["dv_loc"], full["dv_loc"][keys])
    tok = part["cmp_tokens"]
    for k in ("dk_cmp", "dv_cmp", "dscores"):
        np.testing.assert_array_equal(part[k], full[k][tok])


@pytest.mark.parametrize("name", INPUTS)
def test_summary_center_variant_directional_derivatives(name):
    """The summary-centre variant's backward against finite differences of its forward."""
    s, packing = CASES[1][1], "random"
    inp = f64_inputs(s, packing)
    dout = synth.make_dout(s, packing, seed=5).double().numpy()
    grads = oracle.backward(s, inp, dout, center=True)
    rng = np.random.default_rng(23)
    delta = rng.standard_normal(inp[name].shape)
    eps = 1e-6

    def loss_c(x):
        return float(np.sum(oracle.forward(s, x, center=True)["out"] * dout))

    fd = (loss_c(dict(inp, **{name: inp[name] + eps * delta})) -
          loss_c(dict(inp, **{name: inp[name] - eps * delta}))) / (2 * eps)
    an = float(np.sum(grads[GRAD[name]] * delta))
    assert abs(fd - an) <= 1e-6 * max(abs(an), 1e-3), f"{name}: fd {fd!r} vs analytic {an!r}"


def test_summary_center_backward_equals_exact_on_unit_blocks():
    """With 1x1x1 blocks the centre is the token's own site: both forms and their gradients coincide."""
    s = CASES[1][1].replace(bz=1, by=1, bx=1)
    inp = f64_inputs(s, "morton")
    dout = synth.make_dout(s, "morton", seed=5).double().numpy()
    a = oracle.backward(s, inp, dout)
    b = oracle.backward(s, inp, dout, center=True)
    for k in GRAD.values():
        np.testing.assert_allclose(b[k], a[k], rtol=0, atol=1e-12 * max(np.abs(a[k]).max(), 1.0))
