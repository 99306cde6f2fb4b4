"""Benchmark of the PACK3D forward pass on B200: tokens/s, per-stage roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 65k|262k|1m|stress|...]
                    [--impl ours|reference] [--train-only] [--flush write-read|write]

One step = one pass of the whole hot path over one synthetic volume: index
map, block summaries, axial RoPE on Q and K_loc, local attention, query x
summary attention with the gate.  The timed step is one pack3d_forward call
on device buffers, CUDA events around it on the launching stream (the
library runs RoPE on its side stream next to the index map and the
summaries).  A second, staged pass calls the C ABI stage entry points in
turn on one stream with CUDA events between them, so each kernel's live
duration is known (``stages``, ``staged_ms_per_step``).  L2 is
flushed between steps, outside the timed events: a 256 MiB write, then a
256 MiB read of another buffer, so that no input is left in L2 and none of
the flush's dirty lines is written back inside a timed kernel (``--flush
write`` drops the read).  ``e2e``
times pack3d_forward_host, the C-ABI call that takes pinned host buffers
(inputs copied in and the output copied out inside the timed region, the
copies overlapped with the stages by the library).

Under torchrun (N > 1) every rank runs an independent replica of the volume
(the operator is single-GPU; ranks exchange nothing on the data path), the
time is the max over ranks and ``value`` counts every rank's tokens.

``train`` times the training block, pack3d_forward_backward (the forward
pass saving its softmax statistics, then the gradients of <dOut, out> with
respect to every input), on the same volume with dOut drawn N(0,1) per site;
tokens/s there count one forward and one backward per token.

``sizes`` (single-GPU runs of the default workload) times the same stages
on the 262k- and 1M-token volumes, where the stage targets are set, with
their values drawn on the device (same distributions; no parity is taken
from them), each with its own clock record.

``--impl reference`` times the float64 CPU oracle on the host cores on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

from typing import Dict

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "PACK3D fwd tokens/s at 65k/262k/1M tokens, 1 B200; % of tensor/HBM roofline"
WORKLOAD_TEXT = {
    "tiny": "4x8x8 lattice (256 tokens), raster packing, fp32, Hq=2, Hkv=1, d_h=64, blocks 1x4x4 (M=16), window 3x3x3",
    "65k": "16x64x64 lattice (65,536 tokens), Morton packing, bf16, Hq=8, Hkv=2, d_h=64, blocks 1x4x4 (M=4,096), window 3x7x7",
    "262k": "16x128x128 lattice (262,144 tokens), block-contiguous packing, bf16, Hq=8, Hkv=2, d_h=64, blocks 1x4x4 (M=16,384), window 3x7x7",
    "1m": "64x128x128 lattice (1,048,576 tokens), random packing, bf16, Hq=8, Hkv=2, d_h=64, blocks 1x4x4 (M=65,536), window 3x7x7",
    "4m": "64x256x256 lattice (4,194,304 tokens), Morton packing, bf16, Hq=8, Hkv=2, d_h=64, blocks 1x4x4 (M=262,144), window 3x7x7; values drawn on the device",
    "8m": "128x256x256 lattice (8,388,608 tokens), Morton packing, bf16, Hq=8, Hkv=2, d_h=64, blocks 1x4x4 (M=524,288), window 3x7x7; values drawn on the device",
    "stress": "16x64x64 lattice (65,536 tokens), raster packing, bf16, Hq=8, Hkv=2, d_h=64, blocks 1x4x4 (M=4,096), window 3x7x7 (the repacking stress case)",
    "allen": "32x128x64 lattice (262,144 tokens; the shape of the Allen WTC-11 token grid, synthetic values), block-contiguous packing, bf16, Hq=8, Hkv=2, d_h=64, blocks 1x4x4 (M=16,384), window 3x7x7",
}
STAGES = ("index", "summaries", "rope", "local", "summary_attn")
KERNELS_PER_STEP = 7   # 2 fills + index, rope (Q and K), summaries, local, summary attention
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one
# summary_attn_tc_kernel launch per workload, from an ncu capture of that
# workload, with the capture it came from; the summary of the capture is kept
# under profiles/.  Emptied whenever that kernel changes until it is captured
# again (a workload without an entry reports null).
SUMMARY_ATTN_TRAFFIC: Dict[str, tuple] = {
    "65k": (212.882176e6 + 48.153344e6,
            "ncu capture of summary_attn_tc_kernel<0> (one-tile build: 96-summary tiles, two P buffers, 2 of 16 "
            "exponential pairs on the FMA pipe) on the 65k volume (profiles/summary_attn_tc_65k.md)"),
}
# Nominal HBM bandwidth of the part (8 TB/s), reported beside the measured copy peak.
HBM_NOMINAL_GBS = 8000.0
# Volumes timed in the `sizes` block of a default single-GPU run.
SIZES = ("262k", "1m")
SIZE_STEPS = {"262k": (3, 8), "1m": (3, 3)}   # (warm-up, timed) steps

# Launches at least this long are rated against the sustained bf16 peak.
SUSTAINED_MS = 1000.0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def mean_window(s) -> float:
    """Mean clipped window size: product over axes of the mean clipped count."""
    def axis(n, r):
        return float(np.mean([min(n - 1, i + r) - max(0, i - r) + 1 for i in range(n)]))
    return axis(s.Z, s.rz) * axis(s.H, s.ry) * axis(s.W, s.rx)


def algorithmic_work(s):
    """Per-launch algorithmic bytes / flops of each stage: the bytes every stage
    must read and write once (inputs, outputs, the o_loc hand-over) and the
    useful flops of the two attention branches (4 d per query-key pair and
    head; w̄ = the mean clipped window size)."""
    eb = 2 if s.dtype == "bf16" else 4
    d = s.d_h
    N, M = s.N, s.M
    wbar = mean_window(s)
    return {
        "index": {"bytes": N * (12 + 4 + 4)},
        "rope": {"bytes": N * ((s.Hq + s.Hkv) * d * eb * 2 + 12)},
        "summaries": {"bytes": N * (s.Hkv * d * eb * 2 + s.Hkv * 4 + 4) + M * s.Hkv * d * eb * 2},
        "local": {"bytes": N * (s.Hq * d * eb + 2 * s.Hkv * d * eb + s.Hq * d * 4 + 4),
                  "flops": 4.0 * d * s.Hq * N * wbar},
        "summary_attn": {"flops": 4.0 * d * s.Hq * N * M,
                         "bytes": N * (s.Hq * d * eb * 2 + s.Hq * d * 4 + s.Hq * 8) + 2 * M * s.Hkv * d * eb},
    }


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples taken during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def _reduce_device():
    """Device of the tensors the process group reduces: the GPU under NCCL, the host under gloo."""
    import torch.distributed as dist
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (every rank gets it); the replicas' step time."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(tokens_per_rank: int, world: int, ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (ms * 1e-3)


def barrier(world):
    import torch
    if torch.cuda.is_available():
        torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def cpu_oracle_sample(s, inp, target_s: float = 12.0, center: bool = False):
    """Times the oracle on this workload: the whole-volume stages (index map, K_loc
    rotation, summaries) once, the per-query stages on a sample of rows sized to
    about ``target_s`` seconds, extrapolated to all N rows.  Returns a dict."""
    import torch

    import oracle
    t0 = time.perf_counter()
    st, g2p, mem = oracle.build_index(s, inp["coords"])
    coords = inp["coords"].numpy()
    klr = oracle.rotate(s, coords, inp["k_loc"])
    ks, vs = oracle.summaries(s, coords, mem, inp["k_cmp"], inp["v_cmp"], inp["scores"], center=center)
    t_shared = time.perf_counter() - t0

    def per_rows(count, seed):
        rows = synth.sample_rows(s.N, count, seed)
        t = time.perf_counter()
        qr = oracle.rotate(s, coords[rows], inp["q"][torch.from_numpy(rows)])
        ol = oracle.local_attn(s, coords, g2p, qr, klr, inp["v_loc"], rows)
        oc = oracle.summary_attn(s, qr, ks, vs)
        oracle.gate_mix(s, inp["gate"], ol, oc, rows)
        return len(rows), time.perf_counter() - t

    n0, t0r = per_rows(min(64, s.N), 11)
    n1 = int(min(s.N, max(64, n0 * max(0.0, target_s - t_shared) / max(t0r, 1e-6))))
    n1, t1 = per_rows(n1, 12)
    total = t_shared + t1 * s.N / n1
    return {"value": s.N / total, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": (f"float64 C oracle, OpenMP: whole-volume index map, K_loc RoPE and summaries "
                       f"({t_shared:.2f} s) + RoPE/local/summary attention/gate for {n1} of {s.N} query "
                       f"rows ({t1:.2f} s), per-row time extrapolated to all rows"),
            "seconds": t_shared + t1}


def run_reference(args, s):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = synth.make_inputs(s, s.packing, seed=0)
    vals = []
    for _ in range(args.warmup):
        pass  # the oracle has no warm-up state; warm-up steps are not run
    base = None
    for _ in range(args.steps):
        base = cpu_oracle_sample(s, inp, target_s=max(2.0, 60.0 / max(1, args.steps)))
        vals.append(base["value"])
    value = statistics.mean(vals)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": s.N / value * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD_TEXT[args.config], "tokens": s.N},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": base["cores"], "kind": "oracle",
                             "sample": base["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def summary_center_error(p3, s, d, q_rot, members, err, stream, rows: int = 2048):
    """Logit and output error of the summary-centre variant against the exact form, on the GPU
    outside the timed region: both variants' summaries, the logits of a seeded sample of query rows
    against every summary, and the two whole forward outputs."""
    import torch
    out = {}
    ks, vs, outs = {}, {}, {}
    for name, flags in (("exact", 0), ("center", p3.FLAG_SUMMARY_CENTER)):
        cfg = p3.config_from_shape(s, flags)
        k = torch.empty(s.M, s.Hkv, s.d_h, dtype=d["q"].dtype, device=d["q"].device)
        v = torch.empty_like(k)
        p3.build_summaries(cfg, members, d["k_cmp"], d["v_cmp"], d["scores"], k, v, stream)
        ks[name] = k.float()
        op = p3.Pack3D(cfg, d["q"].device)
        outs[name] = op(d["coords"], d["q"], d["k_loc"], d["v_loc"], d["k_cmp"], d["v_cmp"], d["scores"],
                        d["gate"]).float()
        op.check()
    torch.cuda.synchronize()
    rows = max(64, min(rows, (1 << 27) // (s.Hq * s.M)))   # logits of at most 2^27 floats
    gen = torch.Generator(device="cpu").manual_seed(0)
    r = torch.randint(0, s.N, (rows,), generator=gen).to(q_rot.device)
    q = q_rot[r].float()                                              # [rows, Hq, d]
    kv = [(h * s.Hkv) // s.Hq for h in range(s.Hq)]
    le = torch.einsum("rhd,mhd->rhm", q, ks["exact"][:, kv, :]) * s.softmax_scale
    lc = torch.einsum("rhd,mhd->rhm", q, ks["center"][:, kv, :]) * s.softmax_scale
    out["logit_rel_rms"] = float((lc - le).norm() / le.norm())
    out["logit_max_abs_diff"] = float((lc - le).abs().max())
    out["logit_max_abs"] = float(le.abs().max())
    out["out_rel_rms"] = float((outs["center"] - outs["exact"]).norm() / outs["exact"].norm())
    out["query_rows_sampled"] = rows
    return out


def dense_sdpa_ms(s, q_rot, k_rot, v, stream, reps: int = 2) -> Dict:
    """Comparator: dense softmax attention of every token over every token (torch SDPA, bf16, grouped
    kv heads) on the same rotated Q/K and V, timed with CUDA events after one warm-up call."""
    import torch
    from torch.nn.attention import SDPBackend, sdpa_kernel
    # kv heads repeated to the query heads, so the fused flash kernel runs (no N x N score tensor).
    rep_kv = [(h * s.Hkv) // s.Hq for h in range(s.Hq)]
    qt = q_rot.permute(1, 0, 2).unsqueeze(0)
    kt = k_rot[:, rep_kv, :].permute(1, 0, 2).unsqueeze(0)
    vt = v[:, rep_kv, :].permute(1, 0, 2).unsqueeze(0)

    def call():
        with sdpa_kernel(SDPBackend.FLASH_ATTENTION):
            return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=s.softmax_scale)

    try:
        call()
    except RuntimeError as e:
        return {"unavailable": str(e).splitlines()[0][:200]}
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    ms = statistics.mean(ts)
    flops = 4.0 * s.N * s.N * s.d_h * s.Hq
    return {"ms": ms, "tflops": flops / (ms * 1e-3) / 1e12, "calls_timed": reps,
            "what": "torch scaled_dot_product_attention (flash backend), bf16, all N x N pairs, kv heads repeated"}


class L2Flush:
    """Empties L2 between timed steps (outside the timed events): a 256 MiB
    write and, in the default mode, a 256 MiB read of a second buffer, which
    evicts the write's dirty lines so their write-back is not charged to the
    first timed kernel."""

    TEXT = {"write-read": "flushed between steps (256 MiB write, then a 256 MiB read; outside the timed events)",
            "write": "flushed between steps (256 MiB write; outside the timed events)"}

    def __init__(self, dev, mode: str):
        import torch
        self.mode = mode
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.rd = torch.zeros(64 << 20, dtype=torch.int32, device=dev) if mode == "write-read" else None

    def __call__(self):
        import torch
        self.buf.zero_()
        if self.rd is not None:
            torch.sum(self.rd, dtype=torch.int64)

    @property
    def text(self) -> str:
        return self.TEXT[self.mode]


def time_training_block(p3, args, s, cfg, d, inp_host, flush, stream, err, world, rank, dev,
                        device_dout: bool = False) -> Dict:
    """pack3d_forward_backward on the resident inputs: W untimed calls, then K
    timed ones with CUDA events on the launching stream, L2 flushed between
    calls outside the events; the max over ranks."""
    import torch
    if device_dout or args.config in synth.DEVICE_DRAWN:
        gen = torch.Generator(device=dev).manual_seed(rank + 2)
        dout = torch.randn(d["q"].shape, generator=gen, device=dev, dtype=torch.float32).to(d["q"].dtype)
    else:
        dout = synth.make_dout(s, s.packing, seed=rank).to(dev)
    out = torch.empty_like(d["q"])
    grads = p3.empty_grads(d["q"], d["k_loc"], d["scores"], d["gate"])
    tws = torch.empty(p3.train_workspace_bytes(cfg), dtype=torch.uint8, device=dev)
    evs = []
    for k in range(args.warmup + args.steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        p3.forward_backward(cfg, d["coords"], d["q"], d["k_loc"], d["v_loc"], d["k_cmp"], d["v_cmp"], d["scores"],
                            d["gate"], dout, out, grads, tws, err)
        e1.record(stream)
        if k >= args.warmup:
            evs.append((e0, e1))
    torch.cuda.synchronize()
    if p3.check_status(err) != 0:
        raise RuntimeError("device error during the training-block steps")
    ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in evs), world)
    return {"ms_per_step": ms, "tokens_per_s": replica_value(s.N, world, ms),
            "call": "pack3d_forward_backward (forward saving statistics + every input gradient)",
            "dout": "N(0,1) per lattice site", "l2": flush.text}


def run_train_only(args, s):
    """--train-only: the training block alone (no forward legs), one JSON line."""
    import torch

    import geometry_aware_local_b200 as p3

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = p3.config_from_shape(s)
    d = synth.make_inputs_on_device(s, s.packing, seed=rank, device=dev)
    flush = L2Flush(dev, args.flush)
    err = torch.zeros(4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    barrier(world)
    with ClockSampler(local) as clk:
        train = time_training_block(p3, args, s, cfg, d, None, flush, stream, err, world, rank, dev, device_dout=True)
    if rank == 0:
        line = {"metric": "PACK3D forward+backward tokens/s (training block), 1 B200", "value": train["tokens_per_s"],
                "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": train["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": s.dtype, "data": "synthetic (values drawn on the device)",
                "config": {"workload": WORKLOAD_TEXT[args.config], "tokens": s.N, "summaries": s.M,
                           "packing": s.packing}, "train": train,
                "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def stage_fractions(s, st_ms, peaks) -> Dict:
    """Per-stage ms with achieved GB/s and TFLOP/s against the measured peaks (and the nominal HBM)."""
    work = algorithmic_work(s)
    stages = {}
    for name in STAGES:
        t = st_ms[name] * 1e-3
        w = work[name]
        e = {"ms": st_ms[name]}
        if "bytes" in w:
            e["hbm_gbs"] = w["bytes"] / t / 1e9
            e["hbm_frac"] = e["hbm_gbs"] / peaks["hbm_gbs"]
            e["hbm_frac_nominal"] = e["hbm_gbs"] / HBM_NOMINAL_GBS
        if "flops" in w:
            e["tflops"] = w["flops"] / t / 1e12
            e["tensor_frac"] = e["tflops"] / peaks["bf16_tflops"]
            if peaks.get("bf16_tflops_sustained"):
                # against the power-capped sustained GEMM rate, for launches long enough to run capped
                e["tensor_frac_sustained"] = e["tflops"] / peaks["bf16_tflops_sustained"]
        stages[name] = e
    return stages


class StageTimer:
    """One step = the C-ABI stage entry points one after another on one stream, CUDA events between
    the stages on the launching stream."""

    stages = STAGES

    def __init__(self, p3, s, cfg, d, stream, err):
        import torch
        dev, dt = d["q"].device, d["q"].dtype
        self.p3, self.s, self.cfg, self.d, self.stream, self.err = p3, s, cfg, d, stream, err
        self.g2p = torch.empty(s.N, dtype=torch.int32, device=dev)
        self.mem = torch.empty(s.M, s.v, dtype=torch.int32, device=dev)
        self.qr, self.kr = torch.empty_like(d["q"]), torch.empty_like(d["k_loc"])
        self.ks = torch.empty(s.M, s.Hkv, s.d_h, dtype=dt, device=dev)
        self.vs = torch.empty_like(self.ks)
        self.ol = torch.empty(s.N, s.Hq, s.d_h, dtype=torch.float32, device=dev)
        self.out = torch.empty_like(d["q"])

    def step(self, ev):
        import ctypes
        lib, d, sh = self.p3.lib, self.d, self.stream.cuda_stream
        cfgp = ctypes.byref(self.cfg)
        P = lambda t: t.data_ptr()  # noqa: E731
        ev[0].record(self.stream)
        st = lib.pack3d_build_index(cfgp, P(d["coords"]), P(self.g2p), P(self.mem), P(self.err), sh)
        ev[1].record(self.stream)
        st |= lib.pack3d_build_summaries(cfgp, P(self.mem), P(d["k_cmp"]), P(d["v_cmp"]), P(d["scores"]),
                                         P(self.ks), P(self.vs), sh)
        ev[2].record(self.stream)
        st |= lib.pack3d_rope_qk(cfgp, P(d["coords"]), P(d["q"]), P(self.qr), P(d["k_loc"]), P(self.kr), sh)
        ev[3].record(self.stream)
        st |= lib.pack3d_local_attn(cfgp, P(self.g2p), P(self.qr), P(self.kr), P(d["v_loc"]), P(self.ol),
                                    P(self.err), sh)
        ev[4].record(self.stream)
        st |= lib.pack3d_summary_attn(cfgp, P(self.qr), P(self.ks), P(self.vs), P(self.ol), P(d["gate"]),
                                      P(self.out), P(self.err), sh)
        ev[5].record(self.stream)
        if st:
            raise RuntimeError("a PACK3D entry point failed")

    @staticmethod
    def events():
        import torch
        return [torch.cuda.Event(enable_timing=True) for _ in range(6)]

    def run(self, warmup, steps, flush, world, clock_gpu):
        """W untimed steps, then K timed ones (L2 flushed before each, outside the events) inside a
        clock record; returns the mean stage ms, the mean step ms (max over ranks) and the clocks."""
        for _ in range(warmup):
            self.step(self.events())
        if self.p3.check_status(self.err) != 0:
            raise RuntimeError("device error during warm-up")
        evs = [self.events() for _ in range(steps)]
        barrier(world)
        with ClockSampler(clock_gpu) as clk:
            for k in range(steps):
                flush()
                self.step(evs[k])
            barrier(world)
        st_ms = {name: 0.0 for name in self.stages}
        step_ms = []
        for ev in evs:
            for i, name in enumerate(self.stages):
                st_ms[name] += ev[i].elapsed_time(ev[i + 1])
            step_ms.append(ev[0].elapsed_time(ev[-1]))
        if self.p3.check_status(self.err) != 0:
            raise RuntimeError("device error during the timed steps")
        ms = max_over_ranks(sum(step_ms) / len(step_ms), world)
        return {k: v / steps for k, v in st_ms.items()}, ms, clk.summary()


class ForwardTimer(StageTimer):
    """One step = one pack3d_forward call on the device buffers (every stage in one C-ABI call; the
    library runs RoPE on its side stream next to the index map and the summaries), CUDA events on the
    launching stream around it."""

    stages = ()

    def __init__(self, p3, s, cfg, d, stream, err, out):
        import torch
        self.p3, self.s, self.cfg, self.d, self.stream, self.err, self.out = p3, s, cfg, d, stream, err, out
        self.ws = torch.empty(p3.workspace_bytes(cfg), dtype=torch.uint8, device=d["q"].device)

    def step(self, ev):
        d = self.d
        ev[0].record(self.stream)
        self.p3.forward(self.cfg, d["coords"], d["q"], d["k_loc"], d["v_loc"], d["k_cmp"], d["v_cmp"],
                        d["scores"], d["gate"], self.out, self.ws, self.err, stream=self.stream)
        ev[1].record(self.stream)

    @staticmethod
    def events():
        import torch
        return [torch.cuda.Event(enable_timing=True) for _ in range(2)]


def time_sizes(p3, flush, stream, dev, peaks) -> Dict:
    """The `sizes` block: the stages at 262k and 1M tokens (values drawn on the device)."""
    import torch
    res = {}
    for name in SIZES:
        s = synth.CONFIGS[name]
        cfg = p3.config_from_shape(s)
        d = synth.make_inputs_on_device(s, s.packing, seed=0, device=dev)
        err = torch.zeros(4, dtype=torch.int32, device=dev)
        warm, steps = SIZE_STEPS[name]
        timer = StageTimer(p3, s, cfg, d, stream, err)
        st_ms, staged_ms, _ = timer.run(warm, steps, flush, 1, dev.index or 0)
        whole = ForwardTimer(p3, s, cfg, d, stream, err, timer.out)
        _, ms, clocks = whole.run(warm, steps, flush, 1, dev.index or 0)
        stages = stage_fractions(s, st_ms, peaks)
        res[name] = {"workload": WORKLOAD_TEXT[name], "tokens": s.N, "summaries": s.M, "value": s.N / (ms * 1e-3),
                     "unit": "tokens/s", "ms_per_step": ms, "staged_ms_per_step": staged_ms, "steps": steps,
                     "warmup": warm, "stages": stages, "clocks": clocks,
                     "query_x_summary_tensor_frac": stages["summary_attn"]["tensor_frac"],
                     "summaries_hbm_frac": stages["summaries"]["hbm_frac"],
                     "rope_hbm_frac": stages["rope"]["hbm_frac"],
                     "data": "synthetic, values drawn on the device (same distributions as the host recipe)",
                     "l2": flush.text}
        del timer, whole, d
        torch.cuda.empty_cache()
    return res


def time_zslab(p3, name: str, ranks: int, warmup: int, steps: int, flush, dev) -> Dict:
    """The z-slab split of the volume over `ranks` ranks, every rank's kernels run in turn on this
    GPU (zslab.Plan phases; the two NCCL exchanges are replaced by device copies outside the timed
    regions).  Per rank and step: the boundary-row gather, summaries, RoPE and local attention on
    its extended lattice, and the query x summary stage for its tokens, timed with CUDA events."""
    import torch

    from geometry_aware_local_b200 import zslab
    s = synth.CONFIGS[name]
    cfg = p3.config_from_shape(s)
    d = synth.make_inputs_on_device(s, s.packing, seed=0, device=dev)
    plans = []
    for r in range(ranks):
        _, own = zslab.take_slab(d, zslab.make_plan(cfg, r, ranks))
        plan = zslab.Plan(cfg, own["coords"], r, ranks)
        for k, v in plan.inputs().items():
            v.copy_(own[k])
        plans.append(plan)
    del d
    stream = torch.cuda.current_stream(dev)
    per_rank = [[] for _ in plans]
    for it in range(warmup + steps):
        evs = []
        for r, plan in enumerate(plans):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            plan.pack_halo()
            plan.local()
            e1.record(stream)
            evs.append([e0, e1])
        for r, plan in enumerate(plans):             # the halo exchange, as copies
            below, above = plan.halo_views()
            for view, side, peer in ((below, "above", r - 1), (above, "below", r + 1)):
                if view is not None:
                    _, ks, vs = plans[peer].send[side]
                    view[0].copy_(ks)
                    view[1].copy_(vs)
        parts = [plan.summary_part() for plan in plans]
        for plan in plans:                             # the summary all-gather, as copies
            if plan.uneven:
                plan.k_pad.copy_(torch.cat([k for k, _ in parts]))
                plan.v_pad.copy_(torch.cat([v for _, v in parts]))
                p3.gather_rows(plan.compact, plan.k_pad, plan.k_all)
                p3.gather_rows(plan.compact, plan.v_pad, plan.v_all)
            else:
                plan.k_all.copy_(torch.cat([k for k, _ in parts]))
                plan.v_all.copy_(torch.cat([v for _, v in parts]))
        for r, plan in enumerate(plans):
            flush()
            e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e2.record(stream)
            plan.attend()
            e3.record(stream)
            evs[r] += [e2, e3]
        torch.cuda.synchronize()
        if it >= warmup:
            for r, (e0, e1, e2, e3) in enumerate(evs):
                per_rank[r].append(e0.elapsed_time(e1) + e2.elapsed_time(e3))
    for plan in plans:
        if p3.check_status(plan.err) != 0:
            raise RuntimeError("device error in the z-slab ranks")
    ms = [statistics.mean(v) for v in per_rank]
    eb = 2 if s.dtype == "bf16" else 4
    halo = [sum(2 * (b - a) * s.Hkv * s.d_h * eb for (a, b) in (pl.p.halo_below, pl.p.halo_above)) for pl in plans]
    gathered = plans[0].k_all.shape[0] * s.Hkv * s.d_h * eb * 2
    return {"ranks": ranks, "workload": WORKLOAD_TEXT[name], "per_rank_compute_ms": ms,
            "max_rank_compute_ms": max(ms), "halo_bytes_received_per_rank": halo,
            "summary_bytes_all_gathered": gathered, "steps": steps, "warmup": warmup,
            "note": "every rank's kernels timed in turn on one GPU; the NCCL halo exchange and summary "
                    "all-gather are not timed (device copies stand in for them)"}


def run_ours(args, s):
    import torch

    import geometry_aware_local_b200 as p3

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = p3.config_from_shape(s, p3.FLAG_SUMMARY_CENTER if args.summary_center else 0)
    names = ("coords", "q", "k_loc", "v_loc", "k_cmp", "v_cmp", "scores", "gate")
    if args.config in synth.DEVICE_DRAWN:
        # Too large for host draws: values drawn on the device, host copies made for the e2e leg.
        d = synth.make_inputs_on_device(s, s.packing, seed=rank, device=dev)
        inp_host = {k: d[k].cpu() for k in names}
    else:
        inp_host = synth.make_inputs(s, s.packing, seed=rank)
        d = {k: inp_host[k].to(dev) for k in names}
    err = torch.zeros(4, dtype=torch.int32, device=dev)
    flush = L2Flush(dev, args.flush)
    stream = torch.cuda.current_stream(dev)
    # The per-stage split: the stage entry points in turn, events between them.
    timer = StageTimer(p3, s, cfg, d, stream, err)
    st_ms, staged_ms, _ = timer.run(args.warmup, args.steps, flush, world, local)
    qr, kr, mem, out = timer.qr, timer.kr, timer.mem, timer.out
    # The headline step: one pack3d_forward call on the device buffers.
    whole = ForwardTimer(p3, s, cfg, d, stream, err, out)
    _, ms, clock_rec = whole.run(args.warmup, args.steps, flush, world, local)
    value = replica_value(s.N, world, ms)

    # End to end through the public C-ABI call that takes host buffers
    # (pack3d_forward_host): pinned inputs in, output back, copies inside the
    # timed region and overlapped with the stages by the library.
    hin = {k: inp_host[k].pin_memory() for k in names}
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in hin.values())
    d2h = hout.numel() * hout.element_size()
    del whole
    hws = torch.empty(p3.host_workspace_bytes(cfg), dtype=torch.uint8, device=dev)
    pipe = p3.Pipeline()
    e2e = []
    for k in range(args.warmup + args.steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        p3.forward_host(pipe, cfg, hin["coords"], hin["q"], hin["k_loc"], hin["v_loc"], hin["k_cmp"],
                        hin["v_cmp"], hin["scores"], hin["gate"], hout, hws, err)
        e1.record(stream)
        if k >= args.warmup:
            e2e.append((e0, e1))
    torch.cuda.synchronize()
    pipe.close()
    e2e_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in e2e), world)
    if p3.check_status(err) != 0:
        raise RuntimeError("device error during the e2e steps")

    train = None
    if not args.summary_center and not args.no_train and (args.config not in synth.DEVICE_DRAWN or args.train):
        train = time_training_block(p3, args, s, cfg, d, inp_host, flush, stream, err, world, rank, dev)

    peaks = load_peaks()
    stages = stage_fractions(s, st_ms, peaks)
    variant_err = summary_center_error(p3, s, d, qr, mem, err, stream) if args.summary_center else None
    sa = stages["summary_attn"]
    # A launch of a second or more runs under the board's power cap the whole
    # time, like the measured sustained GEMM loop; shorter ones see burst clocks.
    sustained = sa["ms"] >= SUSTAINED_MS and peaks.get("bf16_tflops_sustained")
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    traffic = SUMMARY_ATTN_TRAFFIC.get(args.config)
    roof = {"bound": "tensor", "achieved": sa["tflops"], "peak": peak, "unit": "TFLOP/s",
            "frac": sa["tflops"] / peak, "traffic": traffic[0] if traffic else None,
            "traffic_source": traffic[1] if traffic else "not captured since the kernel last changed",
            "kernel": "summary_attn_tc_kernel" if s.dtype == "bf16" else "summary_attn_simt_kernel",
            "peak_source": peaks["source"] + (" sustained bf16 (MEASURED_PEAKS.json bf16_tflops_sustained)"
                                              if sustained else " burst bf16 (MEASURED_PEAKS.json bf16_tflops)"),
            "frac_of_burst": sa["tflops"] / peaks["bf16_tflops"]}
    if s.dtype != "bf16":
        roof["bound"] = "alu"
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": s.dtype, "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT[args.config], "tokens": s.N, "summaries": s.M,
                       "packing": s.packing,
                       "parallelism": "replicas only" if world > 1 else "single GPU",
                       "summary_form": "summary-centre variant" if args.summary_center
                       else "rotate-before-compress (exact)",
                       "l2": flush.text},
            "e2e": {"value": s.N * world / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": KERNELS_PER_STEP * args.steps,
            "roofline": roof, "stages": stages, "staged_ms_per_step": staged_ms,
            "clocks": clock_rec}
    if variant_err is not None:
        line["summary_center_vs_exact"] = variant_err
    if train is not None:
        line["train"] = train
    # Comparators named by the workloads: a same-window local-only pass at 65k
    # (index map, RoPE and local attention, the stages that pass runs) and a
    # dense-attention run of the same shape at 1M.
    comp = {}
    if args.config == "65k":
        comp["local_only_ms"] = st_ms["index"] + st_ms["rope"] + st_ms["local"]
        comp["local_only_tokens_per_s"] = s.N * world / (comp["local_only_ms"] * 1e-3)
    if args.config == "1m" and not args.no_dense:
        comp["dense_sdpa"] = dense_sdpa_ms(s, qr, kr, d["v_loc"], stream)
        if "ms" in comp["dense_sdpa"]:
            comp["dense_sdpa"]["speedup_of_pack3d"] = comp["dense_sdpa"]["ms"] / ms
    if comp:
        line["comparators"] = comp
    if world == 1 and args.zslab_ranks > 1:
        line["zslab_emulated"] = time_zslab(p3, args.config, args.zslab_ranks, args.warmup, args.steps, flush, dev)
    if world == 1 and args.config == "65k" and not args.no_sizes and not args.summary_center:
        del timer
        torch.cuda.empty_cache()
        line["sizes"] = time_sizes(p3, flush, stream, dev, peaks)
        line["gpu_launches"] += sum(KERNELS_PER_STEP * SIZE_STEPS[n][1] for n in SIZES)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline and args.config not in synth.DEVICE_DRAWN:
            cb = cpu_oracle_sample(s, inp_host, target_s=12.0, center=args.summary_center)
            cb.pop("seconds")
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="65k", choices=sorted(WORKLOAD_TEXT))
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--flush", default="write-read", choices=sorted(L2Flush.TEXT),
                    help="L2 flush between steps: a write then a read (default), or the write alone")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-attention comparator at 1M")
    ap.add_argument("--train", action="store_true",
                    help="also time the training block on the device-drawn 4m / 8m volumes")
    ap.add_argument("--no-train", action="store_true", help="skip the training-block leg")
    ap.add_argument("--no-sizes", action="store_true",
                    help="skip the 262k / 1M stage timings a default single-GPU run adds")
    ap.add_argument("--train-only", action="store_true",
                    help="time only the training block (pack3d_forward_backward), inputs drawn on the device")
    ap.add_argument("--packing", choices=synth.PACKINGS, default=None,
                    help="override the workload's packing (the stress case times all of them)")
    ap.add_argument("--zslab-ranks", type=int, default=0,
                    help="also time the z-slab split of the volume over this many ranks, every rank's "
                         "kernels in turn on this one GPU (the exchanges are not timed)")
    ap.add_argument("--summary-center", action="store_true",
                    help="time the summary-centre variant of the block summaries and report its error "
                         "against the exact rotate-before-compress form")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    s = synth.CONFIGS[args.config]
    if args.packing is not None:
        s = s.replace(packing=args.packing)
    if args.impl == "reference":
        run_reference(args, s)
    elif args.train_only:
        run_train_only(args, s)
    else:
        run_ours(args, s)


if __name__ == "__main__":
    main()
