"""Python binding of libpack3d.so: the PACK3D local-global attention forward pass on B200.

Argument marshalling only: every stage runs in the CUDA kernels behind the C ABI
declared in ``include/pack3d.h`` ("Geometry Matters in Packed 3D Attention",
Key designs 1-3).  Tensors must be CUDA, contiguous and 16-byte aligned; calls
are asynchronous on torch's current stream.  There is no CPU fallback: if the
library was not built, importing the binding raises.

Typical use (packed order throughout; coords are each token's lattice site)::

    import geometry_aware_local_b200 as p3
    cfg = p3.make_config(Z, H, W)    # Hq=8, Hkv=2, d_h=64, 1x4x4 blocks, 3x7x7 window, bf16
    # coords int32 [N,3]; q [N,8,64]; k_loc, v_loc, k_cmp, v_cmp [N,2,64] (bf16);
    # scores float [N,2]; gate float [N,8,2]
    out = p3.attention(cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate)
    out.backward(dout)               # gradients of every float input

``Pack3D(cfg)`` runs the forward pass with a workspace it keeps;
``forward`` / ``forward_backward`` / ``forward_host`` take caller-owned
buffers; the stage entry points (``build_index``, ``rope_qk``,
``build_summaries``, ``local_attn``, ``summary_attn``) run one stage each.
Every wrapper checks its tensors' dtypes and element counts against the
config before calling the library.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpack3d.so")

F32, BF16 = 0, 1
FLAG_SIMT_SUMMARY = 0x1
FLAG_SIMT_LOCAL = 0x2
FLAG_SUMMARY_CENTER = 0x4     # summary-centre variant of the block summaries (include/pack3d.h)
FLAG_DIAG_STALL = 0x8         # diagnostic: each tensor-core kernel withholds one pipeline step (timeout path)
FLAG_SUMMARY_ONE_TILE = 0x10  # force the one-tile build of the tensor-core query x summary kernel
FLAG_SUMMARY_TWO_TILE = 0x20  # force the two-tile build
DEVERR_COORD_RANGE, DEVERR_DUPLICATE, DEVERR_TIMEOUT = 0x1, 0x2, 0x4

STATUS = {0: "OK", 1: "INVALID_ARG", 2: "SHAPE", 3: "ALIGNMENT", 4: "DTYPE", 5: "NOT_PERMUTATION",
          6: "WORKSPACE", 7: "CUDA", 8: "TIMEOUT"}

ENTRY_POINTS = ("pack3d_default_config", "pack3d_validate_config", "pack3d_workspace_bytes",
                "pack3d_build_index", "pack3d_rope", "pack3d_rope_qk", "pack3d_build_summaries", "pack3d_local_attn",
                "pack3d_summary_attn", "pack3d_summary_attn_rows", "pack3d_gather_rows", "pack3d_exp2_fma_eval",
                "pack3d_forward",
                "pack3d_forward_noalloc",
                "pack3d_pipeline_create",
                "pack3d_pipeline_destroy", "pack3d_host_workspace_bytes", "pack3d_forward_host",
                "pack3d_train_workspace_bytes", "pack3d_forward_backward", "pack3d_check_status",
                "pack3d_status_string", "pack3d_backend_info")


class Pack3DError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({_status_string(status)})")


class Config(ctypes.Structure):
    """Mirror of ``pack3d_config``."""
    _fields_ = [("Z", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32),
                ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("d_h", ctypes.c_int32),
                ("m_z", ctypes.c_int32), ("m_y", ctypes.c_int32), ("m_x", ctypes.c_int32),
                ("reserved0", ctypes.c_int32), ("rope_base", ctypes.c_double),
                ("bz", ctypes.c_int32), ("by", ctypes.c_int32), ("bx", ctypes.c_int32),
                ("rz", ctypes.c_int32), ("ry", ctypes.c_int32), ("rx", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("flags", ctypes.c_int32), ("wait_limit_us", ctypes.c_int32),
                ("coord_scale", ctypes.c_double * 3), ("origin", ctypes.c_int32 * 3),
                ("reserved2", ctypes.c_int32)]

    @property
    def N(self) -> int:
        return self.Z * self.H * self.W

    @property
    def M(self) -> int:
        return self.N // (self.bz * self.by * self.bx)

    @property
    def v(self) -> int:
        return self.bz * self.by * self.bx


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python geometry_aware_local_b200/build.py` "
                          "(there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, C = ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(Config)
    sig = {
        "pack3d_default_config": (None, [C, I32, I32, I32]),
        "pack3d_validate_config": (ctypes.c_int, [C]),
        "pack3d_workspace_bytes": (ctypes.c_size_t, [C]),
        "pack3d_build_index": (ctypes.c_int, [C, P, P, P, P, P]),
        "pack3d_rope": (ctypes.c_int, [C, P, P, P, I32, P]),
        "pack3d_rope_qk": (ctypes.c_int, [C, P, P, P, P, P, P]),
        "pack3d_build_summaries": (ctypes.c_int, [C, P, P, P, P, P, P, P]),
        "pack3d_local_attn": (ctypes.c_int, [C, P, P, P, P, P, P, P]),
        "pack3d_summary_attn": (ctypes.c_int, [C, P, P, P, P, P, P, P, P]),
        "pack3d_summary_attn_rows": (ctypes.c_int, [C, ctypes.c_int64, ctypes.c_int64] + [P] * 8),
        "pack3d_gather_rows": (ctypes.c_int, [P, ctypes.c_int64, P, P, ctypes.c_int64, P]),
        "pack3d_exp2_fma_eval": (ctypes.c_int, [P, P, ctypes.c_int64, P]),
        "pack3d_forward": (ctypes.c_int, [C, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P, P]),
        "pack3d_forward_noalloc": (ctypes.c_int, [C, P, P, P, P, P, P, P, P, P, P, P]),
        "pack3d_pipeline_create": (ctypes.c_int, [ctypes.POINTER(P)]),
        "pack3d_pipeline_destroy": (None, [P]),
        "pack3d_host_workspace_bytes": (ctypes.c_size_t, [C]),
        "pack3d_forward_host": (ctypes.c_int, [P, C, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P, P]),
        "pack3d_train_workspace_bytes": (ctypes.c_size_t, [C]),
        "pack3d_forward_backward": (ctypes.c_int, [C] + [P] * 18 + [ctypes.c_size_t, P, P]),
        "pack3d_check_status": (ctypes.c_int, [P, P]),
        "pack3d_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "pack3d_backend_info": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _status_string(st: int) -> str:
    return lib.pack3d_status_string(st).decode()


def backend_info() -> str:
    return lib.pack3d_backend_info().decode()


def make_config(Z: int, H: int, W: int, *, Hq: int = 8, Hkv: int = 2, d_h: int = 64,
                m: Sequence[int] = (11, 11, 10), rope_base: float = 10000.0,
                block: Sequence[int] = (1, 4, 4), radius: Sequence[int] = (1, 3, 3),
                softmax_scale: Optional[float] = None, dtype: str = "bf16", flags: int = 0,
                coord_scale: Sequence[float] = (1.0, 1.0, 1.0), wait_limit_us: int = 0,
                origin: Sequence[int] = (0, 0, 0)) -> Config:
    c = Config()
    c.Z, c.H, c.W = Z, H, W
    c.Hq, c.Hkv, c.d_h = Hq, Hkv, d_h
    c.m_z, c.m_y, c.m_x = m
    c.rope_base = rope_base
    c.bz, c.by, c.bx = block
    c.rz, c.ry, c.rx = radius
    c.softmax_scale = 1.0 / math.sqrt(d_h) if softmax_scale is None else softmax_scale
    c.dtype = BF16 if dtype in ("bf16", BF16) else F32
    c.flags = flags
    c.wait_limit_us = wait_limit_us
    c.coord_scale[:] = [float(x) for x in coord_scale]
    c.origin[:] = [int(x) for x in origin]
    return c


def config_from_shape(s, flags: int = 0, wait_limit_us: int = 0) -> Config:
    """Config from any object with the fields of ``synth.Pack3DShape``."""
    return make_config(s.Z, s.H, s.W, Hq=s.Hq, Hkv=s.Hkv, d_h=s.d_h, m=(s.m_z, s.m_y, s.m_x),
                       rope_base=s.rope_base, block=(s.bz, s.by, s.bx), radius=(s.rz, s.ry, s.rx),
                       softmax_scale=s.softmax_scale, dtype=s.dtype, flags=flags,
                       coord_scale=getattr(s, "coord_scale", (1.0, 1.0, 1.0)), wait_limit_us=wait_limit_us,
                       origin=getattr(s, "origin", (0, 0, 0)))


def validate(cfg: Config) -> int:
    return lib.pack3d_validate_config(ctypes.byref(cfg))


def workspace_bytes(cfg: Config) -> int:
    return lib.pack3d_workspace_bytes(ctypes.byref(cfg))


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("PACK3D kernels take CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("PACK3D kernels take contiguous tensors")
    return t.data_ptr()


# Element type and element count of every tensor argument, from the layouts of
# include/pack3d.h: "T" is the operator's dtype (config.dtype).
_LAYOUT = {
    "coords": ("i32", lambda c: c.N * 3),
    "q": ("T", lambda c: c.N * c.Hq * c.d_h),          # also q_rot, out, dout, dq
    "kv": ("T", lambda c: c.N * c.Hkv * c.d_h),        # k_loc, v_loc, k_cmp, v_cmp, k_rot and their gradients
    "scores": ("f32", lambda c: c.N * c.Hkv),
    "gate": ("f32", lambda c: c.N * c.Hq * 2),
    "g2p": ("i32", lambda c: c.N),
    "members": ("i32", lambda c: c.M * c.v),
    "sum": ("T", lambda c: c.M * c.Hkv * c.d_h),       # k_sum, v_sum
    "o_loc": ("f32", lambda c: c.N * c.Hq * c.d_h),
}


def _check_layout(what: str, cfg, **tensors):
    """Refuses, before anything runs, a tensor whose element type or element count
    does not match the config: the kernels trust the sizes the config implies,
    so a short buffer would be read or written out of bounds.  Arguments are
    given as kind=(name, tensor); None (a nullable argument) and raw integer
    pointers are not checked.  An invalid config is left to the C ABI to report."""
    import torch
    if validate(cfg) != 0:
        return
    types = {"T": torch.bfloat16 if cfg.dtype == BF16 else torch.float32, "f32": torch.float32,
             "i32": torch.int32}
    for kind, items in tensors.items():
        base = kind.rstrip("0123456789")
        if base == "rope":                      # x / y of pack3d_rope: T [N, heads, d_h]
            heads = items[0]
            items = items[1:]
            dt, count = types["T"], cfg.N * heads * cfg.d_h
        else:
            code, size = _LAYOUT[base]
            dt, count = types[code], size(cfg)
        for name, t in items:
            if t is None or isinstance(t, int):
                continue
            if t.dtype != dt:
                raise ValueError(f"{what}: {name} must be {dt}, got {t.dtype}")
            if t.numel() != count:
                raise ValueError(f"{what}: {name} must hold {count} elements for this config, "
                                 f"got {t.numel()} (shape {tuple(t.shape)})")


def _check_err(what: str, err):
    import torch
    if err is not None and not isinstance(err, int) and (err.dtype != torch.int32 or err.numel() < 1):
        raise ValueError(f"{what}: the error word must be an int32 tensor of at least one element")


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(st: int, what: str):
    if st != 0:
        raise Pack3DError(st, what)


def build_index(cfg, coords, g2p, members, err, stream=None):
    _check_layout("build_index", cfg, coords=[("coords", coords)], g2p=[("g2p", g2p)],
                  members=[("members", members)])
    _check_err("build_index", err)
    _check(lib.pack3d_build_index(ctypes.byref(cfg), _ptr(coords), _ptr(g2p), _ptr(members), _ptr(err),
                                  _stream(stream)), "pack3d_build_index")


def rope(cfg, coords, x, y, heads: int, stream=None):
    _check_layout("rope", cfg, coords=[("coords", coords)], rope=[heads, ("x", x), ("y", y)])
    _check(lib.pack3d_rope(ctypes.byref(cfg), _ptr(coords), _ptr(x), _ptr(y), heads, _stream(stream)),
           "pack3d_rope")


def rope_qk(cfg, coords, q, q_rot, k, k_rot, stream=None):
    _check_layout("rope_qk", cfg, coords=[("coords", coords)], q=[("q", q), ("q_rot", q_rot)],
                  kv=[("k", k), ("k_rot", k_rot)])
    _check(lib.pack3d_rope_qk(ctypes.byref(cfg), _ptr(coords), _ptr(q), _ptr(q_rot), _ptr(k), _ptr(k_rot),
                              _stream(stream)), "pack3d_rope_qk")


def build_summaries(cfg, members, k_cmp, v_cmp, scores, k_sum, v_sum, stream=None):
    _check_layout("build_summaries", cfg, members=[("members", members)], kv=[("k_cmp", k_cmp), ("v_cmp", v_cmp)],
                  scores=[("scores", scores)], sum=[("k_sum", k_sum), ("v_sum", v_sum)])
    _check(lib.pack3d_build_summaries(ctypes.byref(cfg), _ptr(members), _ptr(k_cmp), _ptr(v_cmp),
                                      _ptr(scores), _ptr(k_sum), _ptr(v_sum), _stream(stream)),
           "pack3d_build_summaries")


def local_attn(cfg, g2p, q_rot, k_rot, v_loc, o_loc, err=None, stream=None):
    _check_layout("local_attn", cfg, g2p=[("g2p", g2p)], q=[("q_rot", q_rot)], kv=[("k_rot", k_rot), ("v_loc", v_loc)],
                  o_loc=[("o_loc", o_loc)])
    _check_err("local_attn", err)
    _check(lib.pack3d_local_attn(ctypes.byref(cfg), _ptr(g2p), _ptr(q_rot), _ptr(k_rot), _ptr(v_loc),
                                 _ptr(o_loc), _ptr(err), _stream(stream)), "pack3d_local_attn")


def summary_attn(cfg, q_rot, k_sum, v_sum, o_loc, gate, out, err=None, stream=None):
    _check_layout("summary_attn", cfg, q=[("q_rot", q_rot), ("out", out)], sum=[("k_sum", k_sum), ("v_sum", v_sum)],
                  o_loc=[("o_loc", o_loc)], gate=[("gate", gate)])
    _check_err("summary_attn", err)
    _check(lib.pack3d_summary_attn(ctypes.byref(cfg), _ptr(q_rot), _ptr(k_sum), _ptr(v_sum), _ptr(o_loc),
                                   _ptr(gate), _ptr(out), _ptr(err), _stream(stream)), "pack3d_summary_attn")


def summary_attn_rows(cfg, tokens: int, summaries: int, q_rot, k_sum, v_sum, o_loc, gate, out, err=None,
                      stream=None):
    """Stages 4+5 for `tokens` query tokens against `summaries` summaries (pack3d_summary_attn_rows):
    q_rot / out [tokens, Hq, d_h], o_loc [tokens, Hq, d_h] float, gate [tokens, Hq, 2] float,
    k_sum / v_sum [summaries, Hkv, d_h]; the config supplies heads, scale, dtype and flags."""
    import torch
    if validate(cfg) == 0:
        tdt = torch.bfloat16 if cfg.dtype == BF16 else torch.float32
        want = {"q_rot": (tdt, tokens * cfg.Hq * cfg.d_h), "out": (tdt, tokens * cfg.Hq * cfg.d_h),
                "k_sum": (tdt, summaries * cfg.Hkv * cfg.d_h), "v_sum": (tdt, summaries * cfg.Hkv * cfg.d_h),
                "o_loc": (torch.float32, tokens * cfg.Hq * cfg.d_h), "gate": (torch.float32, tokens * cfg.Hq * 2)}
        for name, t in (("q_rot", q_rot), ("out", out), ("k_sum", k_sum), ("v_sum", v_sum), ("o_loc", o_loc),
                        ("gate", gate)):
            if t is None or isinstance(t, int):
                continue
            dt, count = want[name]
            if t.dtype != dt or t.numel() != count:
                raise ValueError(f"summary_attn_rows: {name} must be {dt} with {count} elements, "
                                 f"got {t.dtype} with {t.numel()}")
    _check_err("summary_attn_rows", err)
    _check(lib.pack3d_summary_attn_rows(ctypes.byref(cfg), int(tokens), int(summaries), _ptr(q_rot), _ptr(k_sum),
                                        _ptr(v_sum), _ptr(o_loc), _ptr(gate), _ptr(out), _ptr(err),
                                        _stream(stream)), "pack3d_summary_attn_rows")


def gather_rows(idx, src, dst, stream=None):
    """dst[i] = src[idx[i]] row by row (pack3d_gather_rows); idx int32 [n], src [rows, ...] and dst [n, ...]
    contiguous with the same row shape and dtype; a negative index gives a zero row."""
    import torch
    n = idx.numel()
    same_rows = src.dtype == dst.dtype and tuple(src.shape[1:]) == tuple(dst.shape[1:]) and dst.shape[0] == n
    if idx.dtype != torch.int32 or not same_rows or not all(t.is_contiguous() for t in (idx, src, dst)):
        raise ValueError("gather_rows: idx must be int32 [n], src and dst contiguous rows of one shape and dtype")
    row_bytes = dst[0].numel() * dst.element_size() if n else 16
    _check(lib.pack3d_gather_rows(_ptr(idx), int(n), _ptr(src), _ptr(dst), int(row_bytes), _stream(stream)),
           "pack3d_gather_rows")


def exp2_fma_eval(x, y, stream=None):
    """y = 2^x by the FMA-pipe cubic the one-tile query x summary kernel uses (pack3d_exp2_fma_eval);
    x and y float32 contiguous CUDA tensors of one size."""
    import torch
    if x.dtype != torch.float32 or y.dtype != torch.float32 or x.numel() != y.numel() or \
            not (x.is_contiguous() and y.is_contiguous()):
        raise ValueError("exp2_fma_eval: x and y must be contiguous float32 tensors of one size")
    _check(lib.pack3d_exp2_fma_eval(_ptr(x), _ptr(y), int(x.numel()), _stream(stream)), "pack3d_exp2_fma_eval")


def _check_forward_args(what, cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out, err):
    _check_layout(what, cfg, coords=[("coords", coords)], q=[("q", q), ("out", out)],
                  kv=[("k_loc", k_loc), ("v_loc", v_loc), ("k_cmp", k_cmp), ("v_cmp", v_cmp)],
                  scores=[("scores", scores)], gate=[("gate", gate)])
    _check_err(what, err)


def forward(cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out, workspace, err, stream=None):
    _check_forward_args("forward", cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out, err)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.pack3d_forward(ctypes.byref(cfg), _ptr(coords), _ptr(q), _ptr(k_loc), _ptr(v_loc), _ptr(k_cmp),
                              _ptr(v_cmp), _ptr(scores), _ptr(gate), _ptr(out), _ptr(workspace), ws_bytes,
                              _ptr(err), _stream(stream)), "pack3d_forward")


def forward_noalloc(cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out, err=None, stream=None):
    """pack3d_forward with the library's built-in scratch array instead of a workspace (for
    callers that cannot allocate device memory); see include/pack3d.h for its limit and rules."""
    _check_forward_args("forward_noalloc", cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out, err)
    _check(lib.pack3d_forward_noalloc(ctypes.byref(cfg), _ptr(coords), _ptr(q), _ptr(k_loc), _ptr(v_loc),
                                      _ptr(k_cmp), _ptr(v_cmp), _ptr(scores), _ptr(gate), _ptr(out), _ptr(err),
                                      _stream(stream)), "pack3d_forward_noalloc")


def _host_ptr(t) -> int:
    if t.is_cuda:
        raise ValueError("pack3d_forward_host takes host tensors (page-locked for asynchronous copies)")
    if not t.is_contiguous():
        raise ValueError("PACK3D takes contiguous tensors")
    return t.data_ptr()


def host_workspace_bytes(cfg: Config) -> int:
    return int(lib.pack3d_host_workspace_bytes(ctypes.byref(cfg)))


class Pipeline:
    """The copy streams and events of pack3d_forward_host, bound to the current device."""

    def __init__(self):
        h = ctypes.c_void_p()
        _check(lib.pack3d_pipeline_create(ctypes.byref(h)), "pack3d_pipeline_create")
        self.handle = h

    def close(self):
        if self.handle:
            lib.pack3d_pipeline_destroy(self.handle)
            self.handle = None

    def __del__(self):
        self.close()


def forward_host(pipeline, cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out, workspace, err,
                 stream=None):
    """pack3d_forward from host tensors (inputs and `out`), copies overlapped with the stages; the result
    is in `out` once the stream is synchronised."""
    _check_forward_args("forward_host", cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out, err)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.pack3d_forward_host(pipeline.handle, ctypes.byref(cfg), _host_ptr(coords), _host_ptr(q),
                                   _host_ptr(k_loc), _host_ptr(v_loc), _host_ptr(k_cmp), _host_ptr(v_cmp),
                                   _host_ptr(scores), _host_ptr(gate), _host_ptr(out), _ptr(workspace), ws_bytes,
                                   _ptr(err), _stream(stream)), "pack3d_forward_host")


def train_workspace_bytes(cfg: Config) -> int:
    return int(lib.pack3d_train_workspace_bytes(ctypes.byref(cfg)))


GRAD_NAMES = ("dq", "dk_loc", "dv_loc", "dk_cmp", "dv_cmp", "dscores", "dgate")


def forward_backward(cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, dout, out, grads, workspace, err,
                     stream=None):
    """pack3d_forward_backward: the forward output into `out` and the gradients of <dout, out> into the
    tensors of the dict `grads` (keys GRAD_NAMES, shapes and dtypes of the matching inputs)."""
    _check_forward_args("forward_backward", cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out, err)
    _check_layout("forward_backward", cfg, q=[("dout", dout), ("dq", grads["dq"])],
                  kv=[(k, grads[k]) for k in ("dk_loc", "dv_loc", "dk_cmp", "dv_cmp")],
                  scores=[("dscores", grads["dscores"])], gate=[("dgate", grads["dgate"])])
    ws_bytes = workspace.numel() * workspace.element_size()
    g = [grads[k] for k in GRAD_NAMES]
    _check(lib.pack3d_forward_backward(ctypes.byref(cfg), _ptr(coords), _ptr(q), _ptr(k_loc), _ptr(v_loc),
                                       _ptr(k_cmp), _ptr(v_cmp), _ptr(scores), _ptr(gate), _ptr(dout), _ptr(out),
                                       *[_ptr(x) for x in g], _ptr(workspace), ws_bytes, _ptr(err),
                                       _stream(stream)), "pack3d_forward_backward")


def empty_grads(q, k_loc, scores, gate):
    """Output tensors for forward_backward, shaped like the inputs they differentiate."""
    import torch
    return {"dq": torch.empty_like(q), "dk_loc": torch.empty_like(k_loc), "dv_loc": torch.empty_like(k_loc),
            "dk_cmp": torch.empty_like(k_loc), "dv_cmp": torch.empty_like(k_loc),
            "dscores": torch.empty_like(scores), "dgate": torch.empty_like(gate)}


def check_status(err, stream=None) -> int:
    """Synchronises the stream, reads and clears the device error word; returns the status code."""
    return lib.pack3d_check_status(_ptr(err), _stream(stream))


class Pack3D:
    """Owns the workspace and error word of one configuration on one device."""

    def __init__(self, cfg: Config, device="cuda"):
        import torch
        st = validate(cfg)
        if st != 0:
            raise Pack3DError(st, "pack3d_validate_config")
        self.cfg = cfg
        self.device = torch.device(device)
        self.workspace = torch.empty(workspace_bytes(cfg), dtype=torch.uint8, device=self.device)
        self.err = torch.zeros(4, dtype=torch.int32, device=self.device)

    def __call__(self, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out=None):
        import torch
        if out is None:
            out = torch.empty_like(q)
        forward(self.cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out, self.workspace, self.err)
        return out

    def check(self):
        st = check_status(self.err)
        if st != 0:
            raise Pack3DError(st, "pack3d_forward")


def attention(cfg: Config, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate):
    """The PACK3D operator as a differentiable PyTorch op.

    Forward: pack3d_forward.  Backward: pack3d_forward_backward, which reruns
    the forward to save its softmax statistics and returns the gradients of
    every differentiable input (q, k_loc, v_loc, k_cmp, v_cmp, scores, gate;
    coords is integer).  Tensors are CUDA, contiguous, in the layouts of
    include/pack3d.h; the work runs on the current stream.
    """
    return _Pack3DAutograd.apply(cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate)


def _make_autograd():
    import torch

    class Pack3DAutograd(torch.autograd.Function):
        @staticmethod
        def forward(ctx, cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate):
            st = validate(cfg)
            if st != 0:
                raise Pack3DError(st, "pack3d_validate_config")
            out = torch.empty_like(q)
            ws = torch.empty(workspace_bytes(cfg), dtype=torch.uint8, device=q.device)
            err = torch.zeros(4, dtype=torch.int32, device=q.device)
            forward(cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out, ws, err)
            ctx.cfg = cfg
            ctx.err = err
            ctx.save_for_backward(coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate)
            return out

        @staticmethod
        def backward(ctx, dout):
            coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate = ctx.saved_tensors
            dout = dout.to(q.dtype).contiguous()
            grads = empty_grads(q, k_loc, scores, gate)
            out = torch.empty_like(q)
            ws = torch.empty(train_workspace_bytes(ctx.cfg), dtype=torch.uint8, device=q.device)
            forward_backward(ctx.cfg, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, dout, out, grads, ws,
                             ctx.err)
            st = check_status(ctx.err)
            if st != 0:
                raise Pack3DError(st, "pack3d_forward_backward")
            return (None, None, grads["dq"], grads["dk_loc"], grads["dv_loc"], grads["dk_cmp"], grads["dv_cmp"],
                    grads["dscores"], grads["dgate"])

    return Pack3DAutograd


class _LazyAutograd:
    """Defers the torch import until the differentiable op is first used."""
    _cls = None

    @classmethod
    def apply(cls, *args):
        if cls._cls is None:
            cls._cls = _make_autograd()
        return cls._cls.apply(*args)


_Pack3DAutograd = _LazyAutograd
