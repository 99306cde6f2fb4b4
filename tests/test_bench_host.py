"""Host-side arithmetic of bench.py: the algorithmic work its roofline fractions divide by.

The per-launch bytes and flops of every stage are checked against an
independent count: the mean clipped window by brute force over every lattice
site, and the per-token figures of the 65k workload (bf16, Hq=8, Hkv=2,
d_h=64, M = N/16) written out from the operator's definition.
"""
import itertools
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def brute_mean_window(Z, H, W, rz, ry, rx):
    total = 0
    for z, y, x in itertools.product(range(Z), range(H), range(W)):
        n = 0
        for dz, dy, dx in itertools.product(range(-rz, rz + 1), range(-ry, ry + 1), range(-rx, rx + 1)):
            if 0 <= z + dz < Z and 0 <= y + dy < H and 0 <= x + dx < W:
                n += 1
        total += n
    return total / (Z * H * W)


@pytest.mark.parametrize("dims,radii", [((5, 7, 9), (1, 3, 3)), ((2, 3, 4), (1, 1, 1)), ((1, 8, 4), (1, 3, 2)),
                                        ((6, 2, 11), (2, 0, 3))])
def test_mean_window_is_the_mean_clipped_box(dims, radii):
    s = synth.Pack3DShape(Z=dims[0], H=dims[1], W=dims[2], Hq=2, Hkv=1, rz=radii[0], ry=radii[1], rx=radii[2],
                          bz=1, by=1, bx=1)
    assert bench.mean_window(s) == pytest.approx(brute_mean_window(*dims, *radii), rel=1e-12)


def test_mean_window_of_the_configured_volumes():
    # 3x7x7 window clipped at the volume boundary
    for name, ref in (("65k", 133.43), ("262k", 137.13), ("1m", 141.60)):
        assert bench.mean_window(synth.CONFIGS[name]) == pytest.approx(ref, abs=5e-3)


def test_algorithmic_work_per_token_at_65k():
    s = synth.CONFIGS["65k"]
    w = bench.algorithmic_work(s)
    N, M = s.N, s.M
    assert M * 16 == N
    # index: coords (3 int32) read, g2p and members (one int32 each) written
    assert w["index"]["bytes"] == N * 20
    # RoPE: Q (8 heads) and K_loc (2 heads) of 64 bf16 read and written, coords read
    assert w["rope"]["bytes"] == N * (2 * (8 + 2) * 64 * 2 + 12) == N * 2572
    # summaries: K_cmp and V_cmp (2 heads x 64 bf16 each) and 2 float scores and one
    # member index per token read; k~ and v~ (2 heads x 64 bf16) written per block
    assert w["summaries"]["bytes"] == N * (2 * 2 * 64 * 2 + 2 * 4 + 4) + M * 2 * 2 * 64 * 2
    assert w["summaries"]["bytes"] / N == pytest.approx(556.0)
    # query x summary: S = Q k~^T and O = P v~, 2 d flops each per (query row, summary)
    assert w["summary_attn"]["flops"] == 2 * (2 * 64) * (N * 8) * M
    assert w["summary_attn"]["flops"] / N == pytest.approx(8.39e6, rel=1e-3)
    # local: the same two products over the clipped window
    assert w["local"]["flops"] == pytest.approx(4 * 64 * 8 * N * bench.mean_window(s))


@pytest.mark.parametrize("mode", ["write-read", "write"])
def test_l2_flush_modes(mode):
    f = bench.L2Flush("cpu", mode)
    f()
    assert f.buf.numel() == 256 << 20 and int(f.buf.max()) == 0
    assert (f.rd is not None) == (mode == "write-read")
    assert ("read" in f.text) == (mode == "write-read")
