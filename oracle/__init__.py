"""Float64 CPU oracle for the PACK3D operator ("Geometry Matters in Packed 3D Attention").

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg may use this package; the product path never does.  The
arithmetic lives in ``pack3d_oracle.c`` (plain C, float64, OpenMP over rows);
this module compiles it with the host C compiler and marshals numpy arrays.
It imports nothing from the CUDA package.

Each wrapper names the passage of the pages it follows; the C file restates
the equations and lists the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pack3d_oracle.c")
_LIB = os.path.join(_HERE, "liborc.so")

__all__ = ["build", "threads", "build_index", "rotate", "summaries", "local_attn",
           "summary_attn", "gate_mix", "forward", "as_f64", "rotate_t", "backward"]


def build(force: bool = False) -> str:
    """Compile ``pack3d_oracle.c`` into ``liborc.so`` next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".%d.tmp" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-Wall",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("Z", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32),
                ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("dh", ctypes.c_int32),
                ("mz", ctypes.c_int32), ("my", ctypes.c_int32), ("mx", ctypes.c_int32),
                ("base", ctypes.c_double),
                ("bz", ctypes.c_int32), ("by", ctypes.c_int32), ("bx", ctypes.c_int32),
                ("rz", ctypes.c_int32), ("ry", ctypes.c_int32), ("rx", ctypes.c_int32),
                ("scale", ctypes.c_double), ("cscale", ctypes.c_double * 3),
                ("origin", ctypes.c_double * 3)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        lib.orc_build_index.argtypes = [P, P, P, P]
        lib.orc_build_index.restype = ctypes.c_int
        lib.orc_rotate.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_long]
        lib.orc_summaries.argtypes = [P, P, P, P, P, P, P, P]
        lib.orc_summaries_center.argtypes = [P, P, P, P, P, P, P]
        lib.orc_local_attn.argtypes = [P, P, P, P, P, P, P, ctypes.c_long, P]
        lib.orc_summary_attn.argtypes = [P, P, P, P, ctypes.c_long, ctypes.c_long, P]
        lib.orc_gate_mix.argtypes = [P, P, P, ctypes.c_long, P, P, P]
        L = ctypes.c_long
        lib.orc_rotate_t.argtypes = [P, P, P, P, ctypes.c_int, L]
        lib.orc_gate_backward.argtypes = [P, P, P, L, P, P, P, P, P, P]
        lib.orc_local_attn_backward_q.argtypes = [P, P, P, P, P, P, P, P, L, P, P, P]
        lib.orc_local_attn_backward_kv.argtypes = [P, P, P, P, P, P, P, P, P, P, L, P, P]
        lib.orc_summary_attn_backward_q.argtypes = [P, P, P, P, L, L, P, P, P, P]
        lib.orc_summary_attn_backward_kv.argtypes = [P, P, P, P, L, P, P, P, P, L, P, P]
        lib.orc_summaries_backward.argtypes = [P, P, P, P, P, P, P, P, P, L, P, P, P]
        lib.orc_summaries_center_backward.argtypes = [P, P, P, P, P, P, P, P, L, P, P, P]
        _lib = lib
    return _lib


def threads() -> int:
    """OpenMP threads the oracle runs on (OMP_NUM_THREADS, else all cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    return int(env) if env else (os.cpu_count() or 1)


def _cfg(s, scale: Optional[float] = None) -> _Cfg:
    return _Cfg(s.Z, s.H, s.W, s.Hq, s.Hkv, s.d_h, s.m_z, s.m_y, s.m_x, float(s.rope_base),
                s.bz, s.by, s.bx, s.rz, s.ry, s.rx,
                float(s.softmax_scale if scale is None else scale),
                (ctypes.c_double * 3)(*[float(x) for x in s.coord_scale]),
                (ctypes.c_double * 3)(*[float(x) for x in getattr(s, "origin", (0, 0, 0))]))


def as_f64(x) -> np.ndarray:
    """Contiguous float64 numpy copy of a numpy array or torch tensor (bf16 widened exactly)."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def build_index(s, coords):
    """Bijection check, grid-to-packed map and block membership.

    Key design 1 (coordinate-preserving packings) and Key design 2 (contiguous
    blocks).  Returns ``(status, g2p [N], members [M, v])``; status 0 = ok,
    1 = coordinate out of range, 2 = duplicate coordinate.
    """
    c = _i32(coords)
    g2p = np.empty(s.N, np.int32)
    mem = np.empty((s.M, s.v), np.int32)
    cfg = _cfg(s)
    st = _load().orc_build_index(ctypes.byref(cfg), _ptr(c), _ptr(g2p), _ptr(mem))
    return st, g2p, mem


def rotate(s, coords, x, heads: Optional[int] = None) -> np.ndarray:
    """Axial grid RoPE ``R(c_i) x_i`` per head (Key design 1, equation R(c))."""
    xa = as_f64(x)
    n = xa.shape[0]
    heads = heads if heads is not None else xa.shape[1]
    c = _i32(coords)
    y = np.empty_like(xa)
    cfg = _cfg(s)
    _load().orc_rotate(ctypes.byref(cfg), _ptr(c), _ptr(xa), _ptr(y), heads, n)
    return y


def summaries(s, coords, members, k_cmp, v_cmp, scores, center: bool = False):
    """Rotate-before-compress summaries (Key design 2, equations k~_j^R and v~_j).

    center=True: the summary-centre variant (contribution 2 and "Future Directions" 3 of the
    summary page): the pooled key is left unrotated and rotated once by the block's geometric
    centre (a fractional coordinate); v~ is unchanged."""
    c, m = _i32(coords), _i32(members)
    kc, vc, sc = as_f64(k_cmp), as_f64(v_cmp), as_f64(scores)
    ks = np.empty((s.M, s.Hkv, s.d_h))
    vs = np.empty((s.M, s.Hkv, s.d_h))
    cfg = _cfg(s)
    if center:
        _load().orc_summaries_center(ctypes.byref(cfg), _ptr(m), _ptr(kc), _ptr(vc), _ptr(sc), _ptr(ks),
                                     _ptr(vs))
    else:
        _load().orc_summaries(ctypes.byref(cfg), _ptr(c), _ptr(m), _ptr(kc), _ptr(vc), _ptr(sc),
                              _ptr(ks), _ptr(vs))
    return ks, vs


def _rows(s, rows):
    if rows is None:
        return np.arange(s.N, dtype=np.int64)
    return np.ascontiguousarray(rows, dtype=np.int64)


def local_attn(s, coords, g2p, q_rot, k_rot, v_loc, rows=None, scale=None) -> np.ndarray:
    """Exact local attention over the clipped box window (Key design 3).

    ``q_rot`` holds the rotated queries of ``rows`` (all rows if None), in that
    order; ``k_rot`` and ``v_loc`` hold every token.
    """
    r = _rows(s, rows)
    c, g = _i32(coords), _i32(g2p)
    qa, ka, va = as_f64(q_rot), as_f64(k_rot), as_f64(v_loc)
    if qa.shape[0] != r.shape[0]:
        raise ValueError("q_rot must hold exactly the sampled rows")
    o = np.empty((r.shape[0], s.Hq, s.d_h))
    cfg = _cfg(s, scale)
    _load().orc_local_attn(ctypes.byref(cfg), _ptr(c), _ptr(g), _ptr(qa), _ptr(ka), _ptr(va),
                           _ptr(r), r.shape[0], _ptr(o))
    return o


def summary_attn(s, q_rot, k_sum, v_sum, scale=None) -> np.ndarray:
    """Each row of ``q_rot`` against all M summaries with its own softmax (Key design 3)."""
    qa, ka, va = as_f64(q_rot), as_f64(k_sum), as_f64(v_sum)
    o = np.empty((qa.shape[0], s.Hq, s.d_h))
    cfg = _cfg(s, scale)
    _load().orc_summary_attn(ctypes.byref(cfg), _ptr(qa), _ptr(ka), _ptr(va), ka.shape[0],
                             qa.shape[0], _ptr(o))
    return o


def gate_mix(s, gate, o_loc, o_cmp, rows=None) -> np.ndarray:
    """Tokenwise two-way softmax gate (overall framework, learned mixer)."""
    r = _rows(s, rows)
    ga, la, ca = as_f64(gate), as_f64(o_loc), as_f64(o_cmp)
    out = np.empty_like(la)
    cfg = _cfg(s)
    _load().orc_gate_mix(ctypes.byref(cfg), _ptr(ga), _ptr(r), r.shape[0], _ptr(la), _ptr(ca),
                         _ptr(out))
    return out


def forward(s, inputs: Dict, rows=None, center: bool = False) -> Dict[str, np.ndarray]:
    """The whole operator, stage by stage in the pages' order, for ``rows`` (default all).
    ``center`` selects the summary-centre variant of the summaries.

    ``inputs`` holds ``coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate`` in
    packed order (numpy or torch; bf16 values are widened exactly).  Only the
    sampled rows' queries are rotated and attended; keys, values and summaries
    are built for every token.
    """
    st, g2p, mem = build_index(s, inputs["coords"])
    if st != 0:
        raise ValueError("coordinates are not a bijection onto the lattice (status %d)" % st)
    coords = _i32(inputs["coords"])
    r = _rows(s, rows)
    q = inputs["q"]
    if rows is not None:
        q = q[_torch_index(r)] if hasattr(q, "detach") else np.asarray(q)[r]
    qr = rotate(s, coords[r], q)
    klr = rotate(s, coords, inputs["k_loc"])
    ks, vs = summaries(s, coords, mem, inputs["k_cmp"], inputs["v_cmp"], inputs["scores"], center=center)
    ol = local_attn(s, coords, g2p, qr, klr, inputs["v_loc"], r)
    oc = summary_attn(s, qr, ks, vs)
    gate = inputs["gate"]
    out = gate_mix(s, gate, ol, oc, r)
    return {"out": out, "o_loc": ol, "o_cmp": oc, "q_rot": qr, "k_rot": klr,
            "k_sum": ks, "v_sum": vs, "g2p": g2p, "members": mem, "rows": r}


def _torch_index(r):
    import torch
    return torch.from_numpy(r)


# ---- backward pass of the training block --------------------------------------


def rotate_t(s, coords, y, heads: Optional[int] = None) -> np.ndarray:
    """``R(c_i)^T y_i`` per head: the RoPE backward (the transpose of equation R(c))."""
    ya = as_f64(y)
    n = ya.shape[0]
    heads = heads if heads is not None else ya.shape[1]
    c = _i32(coords)
    x = np.empty_like(ya)
    cfg = _cfg(s)
    _load().orc_rotate_t(ctypes.byref(cfg), _ptr(c), _ptr(ya), _ptr(x), heads, n)
    return x


def _ids(x, n):
    if x is None:
        return np.arange(n, dtype=np.int64)
    return np.ascontiguousarray(x, dtype=np.int64)


def _scatter(a: np.ndarray, idx: np.ndarray) -> np.ndarray:
    full = np.empty_like(a)
    full[idx] = a
    return full


def backward(s, inputs: Dict, dout, keys=None, blocks=None, center: bool = False) -> Dict[str, np.ndarray]:
    """Gradients of L = <dout, out> with respect to every input of the operator.

    The chain rule through the forward stages in reverse: the tokenwise gate
    (overall framework), both attention branches (Key design 3), the
    rotate-before-compress summaries (Key design 2) and the axial RoPE (Key
    design 1).  ``dq`` and ``dgate`` come for every token; ``dk_loc`` and
    ``dv_loc`` for the tokens ``keys`` (default all, in that order); ``dk_cmp``,
    ``dv_cmp`` and ``dscores`` for the members of the summary blocks ``blocks``
    (``cmp_tokens`` = their packed indices, block by block, members in raster
    order), or, with ``blocks=None``, for every token in packed order.
    ``center`` differentiates the summary-centre variant of the summaries.
    """
    lib = _load()
    st, g2p, mem = build_index(s, inputs["coords"])
    if st != 0:
        raise ValueError("coordinates are not a bijection onto the lattice (status %d)" % st)
    coords = _i32(inputs["coords"])
    N, Hq, Hkv, d = s.N, s.Hq, s.Hkv, s.d_h
    allr = np.arange(N, dtype=np.int64)
    cfg = _cfg(s)
    # forward quantities the backward reads
    qr = rotate(s, coords, inputs["q"])
    klr = rotate(s, coords, inputs["k_loc"])
    vl = as_f64(inputs["v_loc"])
    ks, vs = summaries(s, coords, mem, inputs["k_cmp"], inputs["v_cmp"], inputs["scores"], center=center)
    ol = local_attn(s, coords, g2p, qr, klr, vl)
    oc = summary_attn(s, qr, ks, vs)
    # gate
    do = as_f64(dout)
    ga = as_f64(inputs["gate"])
    dgate = np.empty((N, Hq, 2))
    dol = np.empty_like(do)
    doc = np.empty_like(do)
    lib.orc_gate_backward(ctypes.byref(cfg), _ptr(ga), _ptr(allr), N, _ptr(ol), _ptr(oc), _ptr(do),
                          _ptr(dgate), _ptr(dol), _ptr(doc))
    # local branch
    dqr_l = np.empty_like(qr)
    lse_l = np.empty((N, Hq))
    del_l = np.empty((N, Hq))
    lib.orc_local_attn_backward_q(ctypes.byref(cfg), _ptr(coords), _ptr(g2p), _ptr(qr), _ptr(klr), _ptr(vl),
                                  _ptr(dol), _ptr(allr), N, _ptr(dqr_l), _ptr(lse_l), _ptr(del_l))
    kk = _ids(keys, N)
    dklr = np.empty((kk.shape[0], Hkv, d))
    dvl = np.empty_like(dklr)
    lib.orc_local_attn_backward_kv(ctypes.byref(cfg), _ptr(coords), _ptr(g2p), _ptr(qr), _ptr(klr), _ptr(vl),
                                   _ptr(dol), _ptr(lse_l), _ptr(del_l), _ptr(kk), kk.shape[0], _ptr(dklr),
                                   _ptr(dvl))
    # compressed branch
    dqr_c = np.empty_like(qr)
    lse_c = np.empty((N, Hq))
    del_c = np.empty((N, Hq))
    lib.orc_summary_attn_backward_q(ctypes.byref(cfg), _ptr(qr), _ptr(ks), _ptr(vs), s.M, N, _ptr(doc),
                                    _ptr(dqr_c), _ptr(lse_c), _ptr(del_c))
    bb = _ids(blocks, s.M)
    dks = np.empty((bb.shape[0], Hkv, d))
    dvs = np.empty_like(dks)
    lib.orc_summary_attn_backward_kv(ctypes.byref(cfg), _ptr(qr), _ptr(ks), _ptr(vs), N, _ptr(doc),
                                     _ptr(lse_c), _ptr(del_c), _ptr(bb), bb.shape[0], _ptr(dks), _ptr(dvs))
    # summaries
    kc, vc, sc = as_f64(inputs["k_cmp"]), as_f64(inputs["v_cmp"]), as_f64(inputs["scores"])
    nt = bb.shape[0] * s.v
    dkc = np.empty((nt, Hkv, d))
    dvc = np.empty_like(dkc)
    dsc = np.empty((nt, Hkv))
    if center:
        lib.orc_summaries_center_backward(ctypes.byref(cfg), _ptr(mem), _ptr(kc), _ptr(vc), _ptr(sc), _ptr(dks),
                                          _ptr(dvs), _ptr(bb), bb.shape[0], _ptr(dkc), _ptr(dvc), _ptr(dsc))
    else:
        lib.orc_summaries_backward(ctypes.byref(cfg), _ptr(coords), _ptr(mem), _ptr(kc), _ptr(vc), _ptr(sc),
                                   _ptr(dks), _ptr(dvs), _ptr(bb), bb.shape[0], _ptr(dkc), _ptr(dvc), _ptr(dsc))
    cmp_tokens = mem[bb].reshape(-1).astype(np.int64)
    if blocks is None:
        # every token is a member of exactly one block: scatter to packed order
        dkc, dvc, dsc = (_scatter(a, cmp_tokens) for a in (dkc, dvc, dsc))
        cmp_tokens = allr
    # RoPE
    dq = rotate_t(s, coords, dqr_l + dqr_c)
    dk_loc = rotate_t(s, coords[kk], dklr)
    return {"dq": dq, "dk_loc": dk_loc, "dv_loc": dvl, "dk_cmp": dkc, "dv_cmp": dvc, "dscores": dsc,
            "dgate": dgate, "keys": kk, "cmp_tokens": cmp_tokens, "blocks": bb,
            "out": gate_mix(s, inputs["gate"], ol, oc), "lse_loc": lse_l, "lse_cmp": lse_c,
            "dk_sum": dks, "dv_sum": dvs}
