"""The bounded-wait error path of the tensor-core kernels, made to run out on purpose.

Every pipeline wait of the tcgen05 kernels gives up after the config's
wait_limit_us.  PACK3D_FLAG_DIAG_STALL makes each of them withhold one step of
its pipeline (a summary tile's TMA load, a key plane's score MMA), so a wait
that depends on it is certain to run out.  The CTA must then let every load and
MMA it did issue complete, free its tensor memory and return, and the call must
report PACK3D_ERR_TIMEOUT through the error word.  No GPU is faulted or hung:
the waits are bounded (2 ms here) and the kernels return normally.  After the
timed-out call, the same call without the flag on the same stream must be
correct, which shows that the context and the kernels' state survived.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

TIMEOUT = 8          # PACK3D_ERR_TIMEOUT
LIMIT_US = 2000


@pytest.fixture(scope="module")
def p3(cuda_device):
    import geometry_aware_local_b200 as p3
    return p3


def small(**kw):
    base = dict(Z=3, H=12, W=20, Hq=8, Hkv=2, rz=1, ry=3, rx=3, dtype="bf16", value_scale=0.125)
    base.update(kw)
    return synth.Pack3DShape(**base)


def rel_err(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(gpu - ref).max() / max(np.abs(ref).max(), 1e-30))


NAMES = ("coords", "q", "k_loc", "v_loc", "k_cmp", "v_cmp", "scores", "gate")
# (ragged bricks, one summary tile) / (a single 1x4x4 block: one key plane, M = 1) / (several summary
# tiles, four-plane bricks)
SHAPES = {"ragged": small(), "one-block": small(Z=1, H=4, W=4), "m-multi": small(Z=4, H=32, W=40)}


def _forward(p3, cfg, d, err):
    out = torch.empty_like(d["q"])
    ws = torch.empty(p3.workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    p3.forward(cfg, *[d[k] for k in NAMES], out, ws, err)
    return out


@pytest.mark.parametrize("build", [0x10, 0x20], ids=["one-tile", "two-tile"])
@pytest.mark.parametrize("name", list(SHAPES))
def test_forward_times_out_then_recovers(p3, name, build):
    s = SHAPES[name]
    inp = synth.make_inputs(s, "random", seed=31)
    d = {k: inp[k].cuda() for k in NAMES}
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    stalled = p3.config_from_shape(s, p3.FLAG_DIAG_STALL | build, wait_limit_us=LIMIT_US)
    _forward(p3, stalled, d, err)
    assert p3.check_status(err) == TIMEOUT
    # the word was read and cleared; the next call on the stream is a normal one
    out = _forward(p3, p3.config_from_shape(s, build), d, err)
    assert p3.check_status(err) == 0
    ref = oracle.forward(s, inp)["out"]
    assert rel_err(out.cpu().double().numpy(), ref) <= 2e-2


@pytest.mark.parametrize("name", list(SHAPES))
def test_each_tensor_core_stage_reports_its_timeout(p3, name):
    """The local-attention kernel and the query x summary kernel each give up on their own."""
    s = SHAPES[name]
    d = {k: v.cuda() for k, v in synth.make_inputs(s, "random", seed=32).items() if k != "sites"}
    cfg = p3.config_from_shape(s)
    stalled = p3.config_from_shape(s, p3.FLAG_DIAG_STALL, wait_limit_us=LIMIT_US)
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    g2p = torch.empty(s.N, dtype=torch.int32, device="cuda")
    mem = torch.empty(s.M, s.v, dtype=torch.int32, device="cuda")
    p3.build_index(cfg, d["coords"], g2p, mem, err)
    qr, kr = torch.empty_like(d["q"]), torch.empty_like(d["k_loc"])
    p3.rope_qk(cfg, d["coords"], d["q"], qr, d["k_loc"], kr)
    ks = torch.empty(s.M, s.Hkv, 64, dtype=torch.bfloat16, device="cuda")
    vs = torch.empty_like(ks)
    p3.build_summaries(cfg, mem, d["k_cmp"], d["v_cmp"], d["scores"], ks, vs)
    assert p3.check_status(err) == 0          # the stages without pipeline waits ran normally
    ol = torch.empty(s.N, s.Hq, 64, dtype=torch.float32, device="cuda")
    p3.local_attn(stalled, g2p, qr, kr, d["v_loc"], ol, err)
    assert p3.check_status(err) == TIMEOUT
    out = torch.empty_like(d["q"])
    p3.summary_attn(stalled, qr, ks, vs, None, None, out, err)
    assert p3.check_status(err) == TIMEOUT
    # and both again without the flag
    p3.local_attn(cfg, g2p, qr, kr, d["v_loc"], ol, err)
    p3.summary_attn(cfg, qr, ks, vs, ol, d["gate"], out, err)
    assert p3.check_status(err) == 0


@pytest.mark.parametrize("name", ["ragged", "m-multi"])
def test_training_block_times_out_then_recovers(p3, name):
    """pack3d_forward_backward: the forward and the three backward tensor-core kernels all stall."""
    s = SHAPES[name]
    inp = synth.make_inputs(s, "random", seed=33)
    dout = synth.make_dout(s, "random", seed=33)
    d = {k: inp[k].cuda() for k in NAMES}
    do = dout.cuda()
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    res = None
    for flags, expect in ((p3.FLAG_DIAG_STALL, TIMEOUT), (0, 0)):
        cfg = p3.config_from_shape(s, flags, wait_limit_us=LIMIT_US if flags else 0)
        out = torch.empty_like(d["q"])
        grads = p3.empty_grads(d["q"], d["k_loc"], d["scores"], d["gate"])
        ws = torch.empty(p3.train_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
        p3.forward_backward(cfg, *[d[k] for k in NAMES], do, out, grads, ws, err)
        assert p3.check_status(err) == expect
        res = grads
    ref = oracle.backward(s, inp, dout)
    for k in ("dq", "dk_loc", "dv_loc", "dk_cmp", "dv_cmp", "dscores", "dgate"):
        assert rel_err(res[k].cpu().double().numpy(), ref[k]) <= 2e-2, k


def test_cuda_core_paths_ignore_the_stall_flag(p3):
    """Float inputs run on CUDA cores, which have no pipeline waits: the flag changes nothing."""
    s = synth.CONFIGS["tiny"]
    inp = synth.make_inputs(s, "raster", seed=34)
    d = {k: inp[k].cuda() for k in NAMES}
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    out = _forward(p3, p3.config_from_shape(s, p3.FLAG_DIAG_STALL, wait_limit_us=LIMIT_US), d, err)
    assert p3.check_status(err) == 0
    assert rel_err(out.cpu().double().numpy(), oracle.forward(s, inp)["out"]) <= 1e-4
