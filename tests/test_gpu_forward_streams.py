"""pack3d_forward's stream contract, through the C ABI.

Inside one call RoPE runs on a library-owned side stream while the index map
and the summaries run on the caller's stream.  The call must still behave as
if every launch were on the caller's stream: it starts after the work already
queued there (here: copies that replace the inputs just before the call), a
later call on the same workspace does not overwrite the rotated Q / K while
the previous call still reads them, and while the stream is captured into a
CUDA graph every launch stays on it.  Each result must equal, bit for bit,
the same inputs' forward run with the device idle before and after.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

NAMES = ("coords", "q", "k_loc", "v_loc", "k_cmp", "v_cmp", "scores", "gate")
SHAPE = synth.Pack3DShape(Z=16, H=64, W=64, Hq=8, Hkv=2, dtype="bf16", value_scale=0.125, packing="morton")


@pytest.fixture(scope="module")
def setup(cuda_device):
    import geometry_aware_local_b200 as p3
    cfg = p3.config_from_shape(SHAPE)
    sets = []
    for seed in (61, 62):
        inp = synth.make_inputs(SHAPE, SHAPE.packing, seed=seed)
        sets.append({k: inp[k].cuda() for k in NAMES})
    ws = torch.empty(p3.workspace_bytes(cfg), dtype=torch.uint8, device=cuda_device)
    err = torch.zeros(4, dtype=torch.int32, device=cuda_device)
    expect = []
    for d in sets:
        out = torch.empty_like(d["q"])
        torch.cuda.synchronize()
        p3.forward(cfg, *(d[k] for k in NAMES), out, ws, err)
        torch.cuda.synchronize()
        expect.append(out)
    assert p3.check_status(err) == 0
    return p3, cfg, sets, expect, ws, err


def test_forward_waits_for_prior_work_on_its_stream(setup):
    """Inputs overwritten on a side torch stream right before each call, several calls back to back
    on one workspace: every output is the idle-device result of the inputs it was given."""
    p3, cfg, sets, expect, ws, err = setup
    buf = {k: torch.empty_like(sets[0][k]) for k in NAMES}
    side = torch.cuda.Stream()
    outs = []
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for i in range(6):
            for k in NAMES:
                buf[k].copy_(sets[i % 2][k])
            out = torch.empty_like(buf["q"])
            p3.forward(cfg, *(buf[k] for k in NAMES), out, ws, err, stream=side)
            outs.append(out)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert p3.check_status(err) == 0
    for i, out in enumerate(outs):
        assert torch.equal(out, expect[i % 2]), f"call {i}"


def test_forward_captured_in_a_cuda_graph(setup):
    """A captured pack3d_forward (every launch on the capture stream) replays to the eager result."""
    p3, cfg, sets, expect, ws, err = setup
    buf = {k: sets[0][k].clone() for k in NAMES}
    out = torch.empty_like(buf["q"])
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):   # an eager call first, as graph capture wants
        p3.forward(cfg, *(buf[k] for k in NAMES), out, ws, err)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        p3.forward(cfg, *(buf[k] for k in NAMES), out, ws, err)
    for i in (1, 0, 1):
        for k in NAMES:
            buf[k].copy_(sets[i][k])
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, expect[i]), f"replay with input set {i}"
    del g
    assert p3.check_status(err) == 0
