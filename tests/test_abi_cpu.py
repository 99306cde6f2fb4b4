"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point its header declares, validates configs and rejects bad
arguments before launching anything."""
import ctypes
import os
import re

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def p3():
    import geometry_aware_local_b200 as p3
    return p3


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(pack3d_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(p3):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(p3.lib, n), n
    assert set(p3.ENTRY_POINTS) <= set(names)


def test_default_config_matches_pages(p3):
    c = p3.Config()
    p3.lib.pack3d_default_config(ctypes.byref(c), 16, 128, 128)
    assert (c.Hq, c.Hkv, c.d_h, c.m_z, c.m_y, c.m_x) == (8, 2, 64, 11, 11, 10)
    assert (c.bz, c.by, c.bx, c.rz, c.ry, c.rx) == (1, 4, 4, 1, 3, 3)
    assert c.rope_base == 10000.0 and abs(c.softmax_scale - 0.125) < 1e-9
    assert p3.validate(c) == 0


@pytest.mark.parametrize("field,value,status", [
    ("d_h", 128, 2), ("Hq", 6, 2), ("Hkv", 3, 2), ("W", 63, 2), ("bx", 0, 2), ("rz", -1, 2),
    ("m_z", 20, 2), ("dtype", 7, 4), ("softmax_scale", 0.0, 1), ("flags", 0x100, 1), ("reserved0", 1, 1),
    ("flags", 0x40, 1), ("flags", 0x30, 1), ("wait_limit_us", -1, 1),
    ("rope_base", -1.0, 1), ("Z", -1, 2), ("W", -4, 2),
])
def test_validate_rejects(p3, field, value, status):
    c = p3.make_config(16, 64, 64)
    setattr(c, field, value)
    assert p3.validate(c) == status


@pytest.mark.parametrize("field,value", [
    ("flags", 0x8), ("flags", 0x10), ("flags", 0x20), ("flags", 0x8 | 0x20 | 0x4), ("wait_limit_us", 0),
    ("wait_limit_us", 1), ("wait_limit_us", 2_000_000),
])
def test_validate_accepts(p3, field, value):
    """The diagnostic stall, the two forced query x summary builds and any non-negative wait limit."""
    c = p3.make_config(16, 64, 64)
    setattr(c, field, value)
    assert p3.validate(c) == 0


@pytest.mark.parametrize("dims", [(0, 64, 64), (16, 0, 64), (16, 64, 0), (0, 0, 0)])
def test_empty_volume_is_a_no_op(p3, dims):
    """A lattice with a zero extent holds no token: it validates, needs no
    workspace, and every entry point returns PACK3D_OK before reading a pointer
    (all NULL here) or touching the device."""
    c = p3.make_config(*dims)
    assert p3.validate(c) == 0 and c.N == 0 and c.M == 0
    assert p3.workspace_bytes(c) == 0
    assert p3.train_workspace_bytes(c) == 0
    assert p3.host_workspace_bytes(c) == 0
    cp, L = ctypes.byref(c), p3.lib
    assert L.pack3d_build_index(cp, None, None, None, None, None) == 0
    assert L.pack3d_rope(cp, None, None, None, 8, None) == 0
    assert L.pack3d_rope_qk(cp, None, None, None, None, None, None) == 0
    assert L.pack3d_build_summaries(cp, None, None, None, None, None, None, None) == 0
    assert L.pack3d_local_attn(cp, None, None, None, None, None, None, None) == 0
    assert L.pack3d_summary_attn(cp, None, None, None, None, None, None, None, None) == 0
    assert L.pack3d_forward(cp, *[None] * 10, 0, None, None) == 0
    assert L.pack3d_forward_noalloc(cp, *[None] * 11) == 0
    assert L.pack3d_forward_host(None, cp, *[None] * 10, 0, None, None) == 0
    assert L.pack3d_forward_backward(cp, *[None] * 18, 0, None, None) == 0


def test_volume_size_limit(p3):
    """N = Z*H*W must stay below 2^24 tokens."""
    assert p3.validate(p3.make_config(255, 256, 256)) == 0      # 16,711,680 tokens
    assert p3.validate(p3.make_config(256, 256, 256)) == 2      # 2^24


def test_table_limit_and_sizes(p3):
    assert p3.validate(p3.make_config(16, 2048, 2048)) == 2   # rope tables too large for shared memory
    for name in ("tiny", "65k", "262k", "1m"):
        s = synth.CONFIGS[name]
        c = p3.config_from_shape(s)
        assert p3.validate(c) == 0
        eb = 2 if s.dtype == "bf16" else 4
        need = s.N * 4 + s.N * 4 + s.N * (s.Hq + s.Hkv) * 64 * eb + 2 * s.M * s.Hkv * 64 * eb + s.N * s.Hq * 64 * 4
        ws = p3.workspace_bytes(c)
        assert need <= ws <= need + 7 * 1024


def test_host_errors_return_before_launch(p3):
    c = p3.make_config(16, 64, 64)
    lib = p3.lib
    fake = 1 << 20          # never dereferenced: every call below fails validation first
    bad = fake + 8
    cfgp = ctypes.byref(c)
    assert lib.pack3d_build_index(cfgp, None, fake, fake, fake, None) == 1
    assert lib.pack3d_build_index(cfgp, bad, fake, fake, fake, None) == 3
    assert lib.pack3d_rope(cfgp, fake, fake, fake, 0, None) == 1
    assert lib.pack3d_rope(cfgp, fake, bad, fake, 8, None) == 3
    assert lib.pack3d_summary_attn(cfgp, fake, fake, fake, None, fake, fake, None, None) == 1
    ws = p3.workspace_bytes(c)
    args = [fake] * 9
    assert lib.pack3d_forward(cfgp, *args, fake, ws - 1, fake, None) == 6
    assert lib.pack3d_forward(cfgp, *args, fake + 16, ws, fake, None) == 6
    assert lib.pack3d_forward(cfgp, *args, fake, ws, None, None) == 1
    assert lib.pack3d_check_status(None, None) == 1
    # the z-slab entry points: an explicit row count, and the row gather
    assert lib.pack3d_summary_attn_rows(cfgp, -1, 4, fake, fake, fake, None, None, fake, None, None) == 1
    assert lib.pack3d_summary_attn_rows(cfgp, 0, 4, None, None, None, None, None, None, None, None) == 0
    assert lib.pack3d_summary_attn_rows(cfgp, 8, 4, None, fake, fake, None, None, fake, None, None) == 1
    assert lib.pack3d_summary_attn_rows(cfgp, 8, 4, bad, fake, fake, None, None, fake, None, None) == 3
    assert lib.pack3d_summary_attn_rows(cfgp, 1 << 24, 4, fake, fake, fake, None, None, fake, None, None) == 2
    assert lib.pack3d_gather_rows(None, 0, None, None, 16, None) == 0
    assert lib.pack3d_gather_rows(fake, -1, fake, fake, 16, None) == 1
    assert lib.pack3d_gather_rows(fake, 4, fake, fake, 24, None) == 1
    assert lib.pack3d_gather_rows(fake, 4, fake, fake, 16 * (2**31), None) == 1
    assert lib.pack3d_gather_rows(None, 4, fake, fake, 16, None) == 1
    assert lib.pack3d_gather_rows(fake, 4, bad, fake, 16, None) == 3
    assert lib.pack3d_exp2_fma_eval(None, None, 0, None) == 0
    assert lib.pack3d_exp2_fma_eval(fake, fake, -1, None) == 1
    assert lib.pack3d_exp2_fma_eval(None, fake, 4, None) == 1
    # the host-buffer pipeline: no pipeline handle, then a workspace too small for the staging copies
    hws = p3.host_workspace_bytes(c)
    assert hws > ws + 50 * 1024 * 1024
    assert lib.pack3d_forward_host(None, cfgp, *args, fake, hws, fake, None) == 1
    assert lib.pack3d_forward_host(fake, cfgp, *args, fake, ws, fake, None) == 6
    for st in range(9):
        assert lib.pack3d_status_string(st)
    assert b"sm_100a" in lib.pack3d_backend_info()


def test_binding_refuses_host_tensors(p3):
    import torch
    c = p3.make_config(4, 8, 8, Hq=2, Hkv=1, radius=(1, 1, 1), dtype="f32")
    x = torch.zeros(256, 2, 64)
    with pytest.raises(ValueError):
        p3.rope(c, torch.zeros(256, 3, dtype=torch.int32), x, x, 2, stream=0)


def test_binding_checks_layouts_before_anything_runs(p3):
    """A tensor whose element type or count does not match the config is refused by
    the binding before any pointer reaches the library (the kernels trust the
    sizes the config implies)."""
    import torch
    c = p3.make_config(4, 8, 8, Hq=2, Hkv=1, radius=(1, 1, 1), dtype="f32")   # N = 256, M = 16
    N, M = 256, 16

    def f(*shape, dt=torch.float32):
        return torch.zeros(*shape, dtype=dt)

    good = dict(coords=f(N, 3, dt=torch.int32), q=f(N, 2, 64), k_loc=f(N, 1, 64), v_loc=f(N, 1, 64),
                k_cmp=f(N, 1, 64), v_cmp=f(N, 1, 64), scores=f(N, 1), gate=f(N, 2, 2))
    out, err, ws = f(N, 2, 64), f(4, dt=torch.int32), torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA"):        # well-formed: stopped only by the device check
        p3.forward(c, *good.values(), out, ws, err)
    for name, t, msg in [("q", f(N - 1, 2, 64), "elements"), ("k_cmp", f(N, 2, 64), "elements"),
                         ("scores", f(N, 1, dt=torch.float64), "float32"), ("coords", f(N, 3), "int32"),
                         ("gate", f(N, 2), "elements"), ("v_loc", f(N, 1, 64, dt=torch.bfloat16), "float32")]:
        args = dict(good, **{name: t})
        with pytest.raises(ValueError, match=msg):
            p3.forward(c, *args.values(), out, ws, err)
    with pytest.raises(ValueError, match="out"):
        p3.forward(c, *good.values(), f(N, 2, 63), ws, err)
    with pytest.raises(ValueError, match="error word"):
        p3.forward(c, *good.values(), out, ws, f(4))
    with pytest.raises(ValueError, match="members"):
        p3.build_index(c, good["coords"], f(N, dt=torch.int32), f(M, 8, dt=torch.int32), err)
    with pytest.raises(ValueError, match="k_sum"):
        p3.build_summaries(c, f(M, 16, dt=torch.int32), good["k_cmp"], good["v_cmp"], good["scores"],
                           f(M - 1, 1, 64), f(M, 1, 64))
    with pytest.raises(ValueError, match="y"):
        p3.rope(c, good["coords"], good["q"], f(N, 1, 64), 2)
    grads = p3.empty_grads(good["q"], good["k_loc"], good["scores"], good["gate"])
    grads["dgate"] = f(N, 2, 1)
    with pytest.raises(ValueError, match="dgate"):
        p3.forward_backward(c, *good.values(), f(N, 2, 64), out, grads, ws, err)


def test_forward_backward_host_errors(p3):
    c = p3.make_config(16, 64, 64)
    lib = p3.lib
    fake = 1 << 20          # never dereferenced: every call below fails before any launch
    cfgp = ctypes.byref(c)
    tws = p3.train_workspace_bytes(c)
    s = synth.CONFIGS["65k"]
    # forward workspace + stats [N,Hq,4] + float dQ_rot [N,Hq,64] + float dk~, dv~ [M,Hkv,64]
    # + float local dK, dV accumulators [N,Hkv,64]
    need = (p3.workspace_bytes(c) + s.N * s.Hq * 16 + s.N * s.Hq * 64 * 4 + 2 * s.M * s.Hkv * 64 * 4
            + 2 * s.N * s.Hkv * 64 * 4)
    assert need <= tws <= need + 4 * 1024
    args = [fake] * 17       # coords .. dgate
    assert lib.pack3d_forward_backward(cfgp, *args, fake, tws - 1, fake, None) == 6
    assert lib.pack3d_forward_backward(cfgp, *args, fake + 16, tws, fake, None) == 6
    assert lib.pack3d_forward_backward(cfgp, *args, fake, tws, None, None) == 1
    nulls = list(args)
    nulls[8] = None          # dout
    assert lib.pack3d_forward_backward(cfgp, *nulls, fake, tws, fake, None) == 1
    bad = list(args)
    bad[11] = fake + 8       # dk_loc misaligned
    assert lib.pack3d_forward_backward(cfgp, *bad, fake, tws, fake, None) == 3
