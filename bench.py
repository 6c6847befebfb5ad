#!/usr/bin/env python
"""Benchmark: packed rows/s of one MiniMax-H3 transformer-block forward on B200.

Default workload: the full-width single block over the 32768-row packed
sequence (512 text | 30720 video rows of a (30, 32, 32) grid | 1536 audio
rows, no padding), hidden 5376, 56 heads x 128, ffn 14336, one timestep per
row, random-init bf16 weights ~N(0, 0.02) (synthetic data; no checkpoint): the
largest single-block workload, where attention is 55% of the block's flops.
``--workload 2`` / ``--workload 3`` select the 8192-row and the padded
16384-row blocks instead.

A step is one block forward (norm+modulate, QKV + QK-norm + RoPE, attention,
O-projection + gated residual, norm+modulate, W1/W3 + SiLU gate, W2 + gated
residual), in place on the packed hidden stream. The per-forward prologue
(timestep MLP + AdaLN projection) and the layout step run once, before timing.
The line also carries the attention kernel timed alone on the padded
16384-row layout (masked attention: padding rows form their own document),
with its fraction of peak over the valid work.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload C] [--impl reference]

N > 1 runs under torch.distributed.run, one process per GPU; every rank runs
its own replica of the workload (the batch axis is a pure replication axis,
so there is no data-path collective) and the reported time is the maximum
over ranks. ``--impl reference`` times the CPU oracle on bounded samples of
the same workload instead: each step is a sample of query rows run through the
float64 block, with the keys and values of every row formed once beforehand.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import (FULL_DIMS, activations, block_weights, config_layout,  # noqa: E402
                       prologue_weights)

METRIC = "packed rows/s per DiT block fwd (bf16, 1xB200); % of dense bf16 TC peak"
UNIT = "rows/s"
DEFAULT_CFG = 4
_DIMS_TXT = "hidden 5376, 56x128 heads, ffn 14336, per-row timesteps"
WORKLOADS = {
    2: ("full-width MiniMax-H3 block, S=8192 packed rows (512 text | 6144 video (6,32,32) | "
        "1536 audio), no padding, " + _DIMS_TXT),
    3: ("full-width MiniMax-H3 block, S=16384 packed rows (1024 text | 12288 video (12,32,32) | "
        "2560 audio | 512 padding rows in 4 runs, own attention document), " + _DIMS_TXT),
    4: ("full-width MiniMax-H3 block, S=32768 packed rows (512 text | 30720 video (30,32,32) | "
        "1536 audio), no padding, " + _DIMS_TXT),
}
MASKED_CFG = 3
KERNELS = ["norm_modulate_1", "qkv_rope", "attention", "out_residual", "norm_modulate_2",
           "ffn_up", "ffn_down_residual"]


# ------------------------------------------------------------------ work counts

def kernel_bytes(dims, V):
    """Algorithmic DRAM bytes per launch: operands read once, results written once."""
    H, A, Fd = dims.hidden, dims.attn_width, dims.ffn
    norm_bytes = V * (2 * H + 2 * H + 2 * 4 * H)
    gate_resid = V * (2 * H + 2 * H + 4 * H)  # x read + written (bf16), gate row of tmod (fp32)
    return {
        "norm_modulate_1": norm_bytes,
        "qkv_rope": V * H * 2 + 3 * A * H * 2 + 3 * V * A * 2,
        "attention": 3 * V * A * 2 + V * A * 2,
        "out_residual": V * A * 2 + H * A * 2 + gate_resid,
        "norm_modulate_2": norm_bytes,
        "ffn_up": V * H * 2 + 2 * Fd * H * 2 + V * Fd * 2,
        "ffn_down_residual": V * Fd * 2 + H * Fd * 2 + gate_resid,
    }


def kernel_work(dims, V):
    """Algorithmic FLOPs (tensor kernels) or bytes (norm kernels) per launch."""
    H, A, Fd, NH, D = dims.hidden, dims.attn_width, dims.ffn, dims.heads, dims.head_dim
    norm_bytes = V * (2 * H + 2 * H + 2 * 4 * H)  # x in, h out, shift/scale rows of tmod (fp32)
    return {
        "norm_modulate_1": ("hbm", norm_bytes),
        "qkv_rope": ("tensor", 2.0 * V * H * 3 * A),
        "attention": ("tensor", 4.0 * NH * D * float(V) ** 2),
        "out_residual": ("tensor", 2.0 * V * A * H),
        "norm_modulate_2": ("hbm", norm_bytes),
        "ffn_up": ("tensor", 2.0 * V * H * 2 * Fd),
        "ffn_down_residual": ("tensor", 2.0 * V * Fd * H),
    }


def block_flops(dims, V):
    return sum(v for k, (b, v) in kernel_work(dims, V).items() if b == "tensor")


# Source file of each kernel: a DRAM-traffic figure recorded from an ncu capture
# is used only while the SHA-256 of this file still matches the recorded one.
KERNEL_SOURCES = {"norm_modulate_1": "norm.cu", "qkv_rope": "gemm.cu", "attention": "attention.cu",
                  "out_residual": "gemm.cu", "norm_modulate_2": "norm.cu", "ffn_up": "gemm.cu",
                  "ffn_down_residual": "gemm.cu"}
def traffic_file(cfg):
    return os.path.join(ROOT, "profiles", f"dram_traffic_config{cfg}.txt")


def measured_traffic(kernel, cfg=DEFAULT_CFG):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch of `kernel` from the
    committed ncu summary of this workload, or None if none was recorded for the
    kernel's current source."""
    src = os.path.join(ROOT, "audio_generation_b200", "csrc", KERNEL_SOURCES[kernel])
    try:
        with open(src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
        with open(traffic_file(cfg)) as f:
            lines = f.read().splitlines()
    except OSError:
        return None
    for line in lines:
        parts = line.split()
        if len(parts) >= 3 and not line.startswith("#") and parts[0] == kernel \
                and parts[1] == digest:
            return float(parts[2])
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ------------------------------------------------------------------ distributed plumbing

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Maximum of a float over all ranks (identity for a single process)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None) -> None:
    if world <= 1:
        return
    import torch.distributed as dist
    if device is not None and dist.get_backend() == "nccl":
        dist.barrier(device_ids=[device.index])
    else:
        dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle timing

def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OracleSampler:
    """Bounded samples of one block forward of a workload on the CPU oracle.

    Set-up (untimed): the workload's weights and inputs, and the keys and values
    of every row of the sequence. A sample (timed) runs ``rows`` query rows
    through the whole float64 block: their modulation, their own q, k and v,
    attention over all S keys, the output projection, the FFN and both
    residuals. Every row of the block costs the same, and the set-up's keys and
    values are the other rows' share of the work, so rows / sample time
    estimates the block's rows/s on the whole sequence.
    """

    def __init__(self, cfg):
        from oracle import h3_oracle as O  # CPU baseline only
        self.O = O
        self.cfg = cfg
        t0 = time.perf_counter()
        self.dims = dims = FULL_DIMS
        self.L = L = config_layout(cfg)
        self.w = block_weights(dims, cfg, 0)
        pw = prologue_weights(dims, cfg)
        self.x = O.bf16_to_f64(activations(dims, cfg, L.S)[0])

        def tmod_rows(ti, n_chunks):
            return O.timestep_modulation(L.timestep[ti], pw.w_t1, pw.w_t2,
                                         pw.w_proj[:n_chunks * dims.hidden], dims.freq_dim,
                                         dims.hidden).reshape(len(ti), n_chunks, dims.hidden)

        self.tmod_rows = tmod_rows
        self.K, self.V = O.key_value_rows(self.x, self.w, L, tmod_rows, dims)
        self.setup_s = time.perf_counter() - t0
        self.rng = np.random.default_rng([cfg, 31337])

    def sample(self, rows):
        r = np.sort(self.rng.choice(self.L.S, size=rows, replace=False))
        t0 = time.perf_counter()
        self.O.query_rows(self.x, self.w, self.L, self.tmod_rows, self.dims, r, self.K, self.V)
        return time.perf_counter() - t0

    def describe(self, rows, n, secs):
        return (f"float64 NumPy oracle block forward of {rows} random query rows per sample "
                f"({n} samples, {secs:.2f} s each on average) over the {self.L.S}-row config-"
                f"{self.cfg} sequence, keys and values of all rows formed beforehand "
                f"({self.setup_s:.1f} s set-up, not counted)")


def oracle_baseline(cfg, rows, samples):
    """cpu_baseline: a few timed oracle samples of the bench's workload."""
    smp = OracleSampler(cfg)
    smp.sample(max(8, rows // 8))  # untimed warm-up (BLAS threads, caches)
    times = [smp.sample(rows) for _ in range(samples)]
    sec = statistics.median(times)
    return {"value": rows / sec, "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "sample": smp.describe(rows, samples, sum(times) / len(times))}


def run_reference(args, world, rank):
    """The oracle as the reference arm: every step is one bounded CPU sample of
    the workload (``--ref-rows`` query rows through the float64 block)."""
    if rank != 0:
        return 0
    cfg = args.workload
    smp = OracleSampler(cfg)
    for _ in range(args.warmup):
        smp.sample(args.ref_rows)
    times = [smp.sample(args.ref_rows) for _ in range(args.steps)]
    total = sum(times)
    val = args.ref_rows * len(times) / total
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total / len(times) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOADS[cfg], "S": config_layout(cfg).S, "B": 1,
                   "step": f"{args.ref_rows} query rows of the block (bounded sample)"},
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": _cores(), "kind": "oracle",
                         "sample": smp.describe(args.ref_rows, len(times), total / len(times))},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ GPU arm

def run_gpu(args, world, rank, local):
    import torch
    from audio_generation_b200 import h3

    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dims = FULL_DIMS
    d = h3.make_dims(dims)
    cfg = args.workload
    L = config_layout(cfg)
    S, V, B = L.S, L.n_valid, 1

    def to_dev_bits(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(
            torch.bfloat16)

    def to_dev_f32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)

    def to_dev_i32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)

    w = block_weights(dims, cfg, 0)
    pw = prologue_weights(dims, cfg)
    wd = {k: to_dev_bits(getattr(w, k)) for k in ("w_qkv", "q_norm", "k_norm", "w_o", "w13", "w2")}
    wd["ada_table"] = to_dev_f32(w.ada_table)
    cw = h3.make_block_weights(wd["w_qkv"], wd["q_norm"], wd["k_norm"], wd["w_o"], wd["w13"],
                               wd["w2"], wd["ada_table"])
    pos, tags, tidx = to_dev_f32(L.pos), to_dev_i32(L.tags), to_dev_i32(L.t_idx)
    vi, ai, ti = to_dev_i32(L.video_idx), to_dev_i32(L.audio_idx), to_dev_i32(L.text_idx)
    layout = h3.h3_layout_prepare(d, S, L.n_t, pos, tags, tidx, vi, ai, ti)
    # per-forward prologue: tmod for the per-row timesteps
    tws_b = h3.h3_timestep_workspace_size(d, L.n_t)
    tws = torch.empty(tws_b, dtype=torch.uint8, device=device)
    tmod = torch.empty((L.n_t, 6, dims.hidden), dtype=torch.float32, device=device)
    h3.h3_timestep_modulation(d, L.n_t, to_dev_f32(L.timestep), to_dev_f32(pw.w_t1),
                              to_dev_f32(pw.w_t2), to_dev_f32(pw.w_proj), tmod, tws, tws_b)
    del tws
    x_host = torch.from_numpy(activations(dims, cfg, S, B).view(np.int16)).view(
        torch.bfloat16).pin_memory()
    x = x_host.to(device)
    ws_b = h3.h3_workspace_size(d, B, S)
    ws = torch.empty(ws_b, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        h3.h3_block_forward(d, cw, layout, tmod, x, B, ws, ws_b, stream)

    # ---- whole-step timing (device events, max over ranks)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    gpu_id = torch.cuda.get_device_properties(device).uuid
    gpu_id = f"GPU-{gpu_id}" if not str(gpu_id).startswith("GPU-") else str(gpu_id)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize(device)
    with ClockSampler(gpu_id) as clk:
        time.sleep(0.3)  # let the sampler start before the timed region
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(device)
    barrier(world, device)
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, world, device)
    err = h3.h3_layout_error(layout)
    if err != h3.H3_OK:
        raise RuntimeError(f"device error word after timing: {h3.h3_status_string(err)}")
    ms_per_step = ms / args.steps
    value = world * B * S / (ms_per_step / 1e3)

    # ---- end to end through the public API with host buffers: every step copies
    # its input rows from pinned host memory and its result back, double-buffered
    # on two copy streams so step k's copies overlap the compute of its neighbours.
    out_host = [torch.empty_like(x_host).pin_memory() for _ in range(2)]
    xd = [x, torch.empty_like(x)]
    h2d_s, d2h_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n, start_ev=None):
        for k in range(n):
            b = k % 2
            with torch.cuda.stream(h2d_s):
                if k == 0 and start_ev is not None:
                    h2d_s.wait_event(start_ev)
                if k >= 2:
                    h2d_s.wait_event(d2h_done[b])  # buffer b's previous result is out
                xd[b].copy_(x_host, non_blocking=True)
                h2d_done[b].record(h2d_s)
            stream.wait_event(h2d_done[b])
            h3.h3_block_forward(d, cw, layout, tmod, xd[b], B, ws, ws_b, stream)
            comp_done[b].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(comp_done[b])
                out_host[b].copy_(xd[b], non_blocking=True)
                d2h_done[b].record(d2h_s)
        for b in range(min(n, 2)):
            stream.wait_event(d2h_done[(n - 1 - b) % 2])

    e2e_steps(2)
    torch.cuda.synchronize(device)
    barrier(world, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_steps(args.steps, start_ev=e0)
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device) / args.steps
    io_bytes = x_host.numel() * 2

    # ---- per-kernel device time inside a run of steps (for the roofline)
    per = {k: 0.0 for k in KERNELS}
    h, g = ws, None  # workspace views for the single steps
    A, Fd = dims.attn_width, dims.ffn
    hbuf = torch.empty((B, S, dims.hidden), dtype=torch.bfloat16, device=device)
    q = torch.empty((B, dims.heads, S, 128), dtype=torch.bfloat16, device=device)
    k, v = torch.empty_like(q), torch.empty_like(q)
    o = torch.empty((B, S, A), dtype=torch.bfloat16, device=device)
    gbuf = torch.empty((B, S, Fd), dtype=torch.bfloat16, device=device)
    launches = [
        ("norm_modulate_1", lambda: h3.h3_norm_modulate(d, layout, B, 0, x, wd["ada_table"], tmod, hbuf, stream)),
        ("qkv_rope", lambda: h3.h3_qkv_rope(d, layout, B, hbuf, wd["w_qkv"], wd["q_norm"], wd["k_norm"], q, k, v, stream)),
        ("attention", lambda: h3.h3_attention(d, layout, B, q, k, v, o, stream)),
        ("out_residual", lambda: h3.h3_out_residual(d, layout, B, o, wd["w_o"], wd["ada_table"], tmod, x, stream)),
        ("norm_modulate_2", lambda: h3.h3_norm_modulate(d, layout, B, 1, x, wd["ada_table"], tmod, hbuf, stream)),
        ("ffn_up", lambda: h3.h3_ffn_up(d, layout, B, hbuf, wd["w13"], gbuf, stream)),
        ("ffn_down_residual", lambda: h3.h3_ffn_down_residual(d, layout, B, gbuf, wd["w2"], wd["ada_table"], tmod, x, stream)),
    ]
    reps = max(3, min(20, args.steps))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(launches) + 1)]
           for _ in range(reps)]
    for _, fn in launches:
        fn()
    for r in range(reps):
        evs[r][0].record(stream)
        for i, (_, fn) in enumerate(launches):
            fn()
            evs[r][i + 1].record(stream)
    torch.cuda.synchronize(device)
    for r in range(reps):
        for i, (name, _) in enumerate(launches):
            per[name] += evs[r][i].elapsed_time(evs[r][i + 1]) / reps
    work = kernel_work(dims, V)
    peaks = load_peaks()
    # Kernels timed inside and right after a run of block steps: when the SM
    # clock sampled over the timed steps sits below 90 % of its maximum (the
    # board at its power cap) or the steps ran for a second or more, the
    # kernels ran in the sustained power state and their tensor peak is the
    # sustained cuBLAS figure; otherwise the burst one. Both fractions are given.
    clocks = clk.summary()
    capped = (clocks.get("sm_mhz") is not None and clocks.get("sm_max_mhz")
              and clocks["sm_mhz"] < 0.9 * clocks["sm_max_mhz"])
    long_run = args.steps * ms_per_step >= 1000.0 or bool(capped)
    tc_peak = peaks["bf16_tflops_sustained"] if long_run else peaks["bf16_tflops"]
    peak_kind = "sustained" if long_run else "burst"
    dom = max(per, key=lambda n: per[n])
    bound, amount = work[dom]
    if bound == "tensor":
        achieved = amount / (per[dom] * 1e-3) / 1e12
        peak, unit = tc_peak, "TFLOP/s"
    else:
        achieved = amount / (per[dom] * 1e-3) / 1e9
        peak, unit = peaks["hbm_gbs"], "GB/s"
    kernels = {}
    for n in KERNELS:
        b, amt = work[n]
        t = per[n] * 1e-3
        if b == "tensor":
            kernels[n] = {"ms": round(per[n], 4), "tflops": round(amt / t / 1e12, 1),
                          "frac_of_peak": round(amt / t / 1e12 / tc_peak, 3)}
        else:
            kernels[n] = {"ms": round(per[n], 4), "gbs": round(amt / t / 1e9, 1),
                          "frac_of_peak": round(amt / t / 1e9 / peaks["hbm_gbs"], 3)}
    flops = block_flops(dims, V)
    del hbuf, q, k, v, o, gbuf
    masked = None if args.no_masked else masked_attention(h3, d, dims, device, stream, peaks)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded random-init weights and activations)",
        "config": {"workload": WORKLOADS[cfg], "S": S, "B": B, "valid_rows": V,
                   "l2": (f"inputs larger than L2 (770 MB of block weights + "
                          f"{L.n_t * 6 * dims.hidden * 4 / 2**30:.1f} GiB tmod per step)"),
                   "parallelism": f"replicas x{world}, no collective on the data path"},
        "tflops": flops / (ms_per_step * 1e-3) / 1e12,
        "frac_of_peak": flops / (ms_per_step * 1e-3) / 1e12 / tc_peak,
        "frac_of_burst_peak": flops / (ms_per_step * 1e-3) / 1e12 / peaks["bf16_tflops"],
        "peak_source": peaks["source"],
        "roofline": {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak,
                     "unit": unit, "frac": achieved / peak, "traffic": measured_traffic(dom, cfg),
                     "peak_kind": peak_kind if bound == "tensor" else "copy",
                     "frac_of_burst": (achieved / peaks["bf16_tflops"] if bound == "tensor"
                                       else achieved / peak),
                     "clock_sm_mhz": clocks.get("sm_mhz"),
                     "algorithmic_bytes": kernel_bytes(dims, V)[dom]},
        "kernels": kernels,
        "attention_masked": masked,
        "e2e": {"value": world * B * S / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": io_bytes, "d2h_bytes_per_step": io_bytes},
        "gpu_launches": len(launches) * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_stack:
        # the 50-block stack over the padded 16384-row layout, two timed forwards
        del x_host, out_host, xd, ws
        torch.cuda.empty_cache()
        st = stack_measure(2, 1, reduce_blocks=(3, 39))
        line["stack_config5"] = {k: st[k] for k in ("value", "unit", "ms_per_step", "tflops",
                                                    "frac_of_sustained_peak", "frac_of_burst_peak",
                                                    "clocks", "steps", "warmup", "token_reduced")}
        line["stack_config5"]["workload"] = st["config"]["workload"]
        torch.cuda.empty_cache()
        # the same stack with every GEMM on e4m3 operands, and the 8-bit block
        s8 = stack_measure(2, 1, e4m3=True)
        line["stack_config5_e4m3"] = {k: s8[k] for k in ("value", "unit", "ms_per_step", "tflops",
                                                         "dtype", "clocks")}
        torch.cuda.empty_cache()
        b8 = e4m3_measure(10, 3, cfg)
        line["block_e4m3"] = {k: b8[k] for k in ("value", "unit", "ms_per_step", "tflops", "dtype",
                                                 "clocks", "qkv_w13_only")}
        torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_baseline(cfg, args.ref_rows, 3)
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    layout.close()
    return 0


def attention_only(h3, d, dims, device, stream, peaks, cfg, reps, warmup=3):
    """The attention kernel alone on one workload's layout (Q, K, V seeded
    N(0, 1) bf16, the scale of q and k after the per-head RMSNorm); only the
    layout tables, q, k, v and o are on the device. Mean time and TFLOP/s over
    the valid work, 4 NH D V^2 (the padding document is not counted)."""
    import torch
    L = config_layout(cfg)
    S, V = L.S, L.n_valid
    to_i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
    pos = torch.from_numpy(np.ascontiguousarray(L.pos, dtype=np.float32)).to(device)
    layout = h3.h3_layout_prepare(d, S, L.n_t, pos, to_i32(L.tags), to_i32(L.t_idx),
                                  to_i32(L.video_idx), to_i32(L.audio_idx), to_i32(L.text_idx))
    g = torch.Generator(device=device)
    g.manual_seed(3003)
    shape = (1, dims.heads, S, dims.head_dim)
    q, k, v = (torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(
        torch.bfloat16) for _ in range(3))
    o = torch.empty((1, S, dims.attn_width), dtype=torch.bfloat16, device=device)
    for _ in range(warmup):
        h3.h3_attention(d, layout, 1, q, k, v, o, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    e0.record(stream)
    for _ in range(reps):
        h3.h3_attention(d, layout, 1, q, k, v, o, stream)
    e1.record(stream)
    torch.cuda.synchronize(device)
    if h3.h3_layout_error(layout) != h3.H3_OK:
        raise RuntimeError("device error word set during the attention run")
    layout.close()
    ms = e0.elapsed_time(e1) / reps
    tf = 4.0 * dims.heads * dims.head_dim * float(V) ** 2 / (ms * 1e-3) / 1e12
    return {"workload": WORKLOADS.get(cfg, CONFIG_NAMES_SHORT.get(cfg)), "S": S,
            "valid_rows": V, "launches": reps, "ms": round(ms, 4), "tflops_valid": round(tf, 1),
            "frac_of_peak": round(tf / peaks["bf16_tflops"], 3), "peak_kind": "burst",
            "frac_of_sustained_peak": round(tf / peaks["bf16_tflops_sustained"], 3)}


CONFIG_NAMES_SHORT = {5: "the 16384-row padded layout of the 50-block stack"}


def run_attention_only(args):
    """--attention-only: the attention kernel alone on the workload's layout
    (own JSON line); with little on the device, for profiler captures."""
    import torch
    from audio_generation_b200 import h3
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    dims = FULL_DIMS
    res = attention_only(h3, h3.make_dims(dims), dims, device, torch.cuda.current_stream(device),
                         load_peaks(), args.workload, args.steps, args.warmup)
    print(json.dumps(dict(res, metric="attention TFLOP/s over the valid work (bf16, 1xB200)",
                          unit="TFLOP/s", value=res["tflops_valid"])))
    return 0


def masked_attention(h3, d, dims, device, stream, peaks, reps=10):
    """The attention kernel alone on the padded 16384-row layout (512 padding
    rows in four runs; two runs straddle a 128-row tile, so two tiles need the
    per-key mask and two are skipped whole), through attention_only."""
    return attention_only(h3, d, dims, device, stream, peaks, MASKED_CFG, reps)


STACK_CFG = 5
STACK_BLOCKS = 50
STACK_WORKLOAD = ("full-width MiniMax-H3 50-block stack forward, S=16384 packed rows (15872 "
                  "valid: text | video | audio with four 128-row padding runs), two timesteps, "
                  "fp32 residual stream inside the stack")


def run_stack(args):
    """--stack: the 50-block stack forward on one GPU, one JSON line; with
    --reduced also the token-reduced stack (blocks [3, 39) on the reduced
    sequence, the page's schedule)."""
    print(json.dumps(stack_measure(args.steps, args.warmup,
                                   (3, 39) if args.reduced else None, e4m3=args.e4m3)))
    return 0


def stack_measure(steps, warmup, reduce_blocks=None, e4m3=False):
    """The 50-block stack forward on one GPU (layout prepared once, the
    per-forward prologue for the two timesteps, then the stack with the valid rows
    gathered into an fp32 stream and scattered back): forward time, valid rows/s
    and TFLOP/s (algorithmic flops of 50 blocks over the valid rows and the valid
    document). With ``reduce_blocks = (r0, r1)`` the stack runs blocks [r0, r1)
    on the token-reduced sequence (h3_stack_forward_reduced: pairs of adjacent
    target-video rows, the video rows of frames t >= 1, merged), and the line
    reports the plain stack's time beside it. With ``e4m3`` every block runs its
    four GEMMs on e4m3 operands (h3_stack_forward_e4m3; weights quantized once,
    before timing)."""
    import torch
    from audio_generation_b200 import h3

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    dims = FULL_DIMS
    d = h3.make_dims(dims)
    L = config_layout(STACK_CFG)
    S, V = L.S, L.n_valid

    def to_dev_bits(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(
            torch.bfloat16)

    def to_dev_f32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)

    def to_dev_i32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)

    keep, cws, w8s = [], [], []
    for i in range(STACK_BLOCKS):
        w = block_weights(dims, STACK_CFG, i)
        t = {k: to_dev_bits(getattr(w, k)) for k in ("w_qkv", "q_norm", "k_norm", "w_o", "w13",
                                                    "w2")}
        t["ada_table"] = to_dev_f32(w.ada_table)
        keep.append(t)
        cws.append(h3.make_block_weights(t["w_qkv"], t["q_norm"], t["k_norm"], t["w_o"],
                                         t["w13"], t["w2"], t["ada_table"]))
        if e4m3:
            q = {}
            for name in ("w_qkv", "w13", "w_o", "w2"):
                rows, K = getattr(w, name).shape
                q[name] = (torch.empty((rows, K), dtype=torch.uint8, device=device),
                           torch.empty(rows, dtype=torch.float32, device=device))
                h3.h3_quantize_e4m3_rows(t[name], rows, K, q[name][0], q[name][1])
            t["q8"] = q
            w8s.append(h3.make_block_weights_e4m3(*q["w_qkv"], *q["w13"], *q["w_o"], *q["w2"]))
    pw = prologue_weights(dims, STACK_CFG)
    pos, tags, tidx = to_dev_f32(L.pos), to_dev_i32(L.tags), to_dev_i32(L.t_idx)
    vi, ai, ti = to_dev_i32(L.video_idx), to_dev_i32(L.audio_idx), to_dev_i32(L.text_idx)
    layout = h3.h3_layout_prepare(d, S, L.n_t, pos, tags, tidx, vi, ai, ti)
    t_dev, w1, w2p, wp = (to_dev_f32(L.timestep), to_dev_f32(pw.w_t1), to_dev_f32(pw.w_t2),
                          to_dev_f32(pw.w_proj))
    tws_b = h3.h3_timestep_workspace_size(d, L.n_t)
    tws = torch.empty(tws_b, dtype=torch.uint8, device=device)
    tmod = torch.empty((L.n_t, 6, dims.hidden), dtype=torch.float32, device=device)
    x_host = torch.from_numpy(activations(dims, STACK_CFG, S, 1).view(np.int16)).view(
        torch.bfloat16)
    x0 = x_host.to(device)
    x = torch.empty_like(x0)
    ws_b = (h3.h3_workspace_size_e4m3 if e4m3 else h3.h3_workspace_size)(d, 1, S)
    ws = torch.empty(ws_b, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def forward():
        x.copy_(x0, non_blocking=True)
        h3.h3_timestep_modulation(d, L.n_t, t_dev, w1, w2p, wp, tmod, tws, tws_b, stream)
        if e4m3:
            h3.h3_stack_forward_e4m3(d, cws, w8s, layout, tmod, x, 1, ws, ws_b, stream)
        else:
            h3.h3_stack_forward(d, cws, layout, tmod, x, 1, ws, ws_b, stream)

    gpu_id = torch.cuda.get_device_properties(device).uuid
    gpu_id = f"GPU-{gpu_id}" if not str(gpu_id).startswith("GPU-") else str(gpu_id)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(gpu_id) as clk:
            time.sleep(0.3)
            e0.record(stream)
            for _ in range(steps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize(device)
        if h3.h3_layout_error(layout) != h3.H3_OK:
            raise RuntimeError("device error word set during the stack run")
        return e0.elapsed_time(e1) / steps, clk

    reduced = None
    if reduce_blocks is not None:
        r0, r1 = reduce_blocks
        target = ((L.tags == 0) & (L.pos[:, 0] >= 1)).astype(np.int32)
        red = h3.h3_layout_reduce(d, layout, to_dev_i32(target))
        rws_b = h3.h3_stack_reduced_workspace_size(d, layout, red, 1)
        rws = torch.empty(rws_b, dtype=torch.uint8, device=device)

        def forward_reduced():
            x.copy_(x0, non_blocking=True)
            h3.h3_timestep_modulation(d, L.n_t, t_dev, w1, w2p, wp, tmod, tws, tws_b, stream)
            h3.h3_stack_forward_reduced(d, cws, layout, red, r0, r1, tmod, x, 1, rws, rws_b,
                                        stream)

        ms_red, clk_red = timed(forward_reduced)
        reduced = {"ms_per_step": ms_red, "value": V / (ms_red * 1e-3), "r0": r0, "r1": r1,
                   "target_rows": int(target.sum()), "clocks": clk_red.summary()}
        red.close()
        del rws
    ms, clk = timed(forward)
    flops = STACK_BLOCKS * block_flops(dims, V)
    peaks = load_peaks()
    tflops = flops / (ms * 1e-3) / 1e12
    line = {
        "metric": "valid packed rows/s per 50-block stack forward (%s, 1xB200)" % (
            "e4m3 GEMM operands" if e4m3 else "bf16"),
        "value": V / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": steps,
        "warmup": warmup, "ms_per_step": ms, "higher_is_better": True,
        "dtype": "e4m3 (QKV, O, W1||W3, W2) + bf16 (attention)" if e4m3 else "bf16",
        "data": "synthetic (seeded random-init weights and activations)",
        "config": {"workload": STACK_WORKLOAD, "S": S, "valid_rows": V, "blocks": STACK_BLOCKS,
                   "n_t": int(L.n_t)},
        "tflops": tflops, "clocks": clk.summary(),
        # prologue, gather / scatter, blocks (two row-quantizing passes more in 8 bits)
        "gpu_launches": steps * (4 + 2 + (9 if e4m3 else 7) * STACK_BLOCKS),
    }
    # fractions of the bf16 peaks (an 8-bit stack's flops are counted as the
    # bf16 stack's, so its fractions can exceed 1)
    pre = "frac_of_bf16_" if e4m3 else "frac_of_"
    line[pre + "sustained_peak"] = tflops / peaks["bf16_tflops_sustained"]
    line[pre + "burst_peak"] = tflops / peaks["bf16_tflops"]
    if reduced is not None:
        reduced["speedup_vs_full_stack"] = ms / reduced["ms_per_step"]
        line["token_reduced"] = reduced
    layout.close()
    return line


def e4m3_measure(steps, warmup, cfg):
    """--e4m3: the block step of the workload with all four GEMMs (QKV, O,
    W1 || W3, W2) on e4m3 operands (h3_block_forward_e4m3; weights quantized once,
    before timing; o and g quantized per row inside the step), and the form with
    only QKV and W1 || W3 in 8 bits beside it. Own JSON line; TFLOP/s over the
    same algorithmic flops as the bf16 block."""
    import torch
    from audio_generation_b200 import h3

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    dims = FULL_DIMS
    d = h3.make_dims(dims)
    L = config_layout(cfg)
    S, V = L.S, L.n_valid
    bits = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(
        torch.bfloat16)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
    w = block_weights(dims, cfg, 0)
    wd = {k: bits(getattr(w, k)) for k in ("w_qkv", "q_norm", "k_norm", "w_o", "w13", "w2")}
    wd["ada_table"] = f32(w.ada_table)
    cw = h3.make_block_weights(wd["w_qkv"], wd["q_norm"], wd["k_norm"], wd["w_o"], wd["w13"],
                               wd["w2"], wd["ada_table"])
    q8 = {}
    for name in ("w_qkv", "w13", "w_o", "w2"):
        rows, K = getattr(w, name).shape
        q8[name] = (torch.empty((rows, K), dtype=torch.uint8, device=device),
                    torch.empty(rows, dtype=torch.float32, device=device))
        h3.h3_quantize_e4m3_rows(wd[name], rows, K, q8[name][0], q8[name][1])
    w8_two = h3.make_block_weights_e4m3(q8["w_qkv"][0], q8["w_qkv"][1], q8["w13"][0],
                                        q8["w13"][1])
    w8 = h3.make_block_weights_e4m3(q8["w_qkv"][0], q8["w_qkv"][1], q8["w13"][0], q8["w13"][1],
                                    q8["w_o"][0], q8["w_o"][1], q8["w2"][0], q8["w2"][1])
    layout = h3.h3_layout_prepare(d, S, L.n_t, f32(L.pos), i32(L.tags), i32(L.t_idx),
                                  i32(L.video_idx), i32(L.audio_idx), i32(L.text_idx))
    pw = prologue_weights(dims, cfg)
    tws_b = h3.h3_timestep_workspace_size(d, L.n_t)
    tws = torch.empty(tws_b, dtype=torch.uint8, device=device)
    tmod = torch.empty((L.n_t, 6, dims.hidden), dtype=torch.float32, device=device)
    h3.h3_timestep_modulation(d, L.n_t, f32(L.timestep), f32(pw.w_t1), f32(pw.w_t2),
                              f32(pw.w_proj), tmod, tws, tws_b)
    del tws
    x = bits(activations(dims, cfg, S, 1))
    ws_b = h3.h3_workspace_size_e4m3(d, 1, S)
    ws = torch.empty(ws_b, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step(ww=w8):
        h3.h3_block_forward_e4m3(d, cw, ww, layout, tmod, x, 1, ws, ws_b, stream)

    # the form with QKV and W1 || W3 only, timed first
    for _ in range(warmup):
        step(w8_two)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step(w8_two)
    t1.record(stream)
    torch.cuda.synchronize(device)
    ms_two = t0.elapsed_time(t1) / steps
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    gpu_id = torch.cuda.get_device_properties(device).uuid
    gpu_id = f"GPU-{gpu_id}" if not str(gpu_id).startswith("GPU-") else str(gpu_id)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id) as clk:
        time.sleep(0.3)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(device)
    if h3.h3_layout_error(layout) != h3.H3_OK:
        raise RuntimeError("device error word set during the e4m3 run")
    ms = e0.elapsed_time(e1) / steps
    tflops = block_flops(dims, V) / (ms * 1e-3) / 1e12
    peaks = load_peaks()
    line = {
        "metric": METRIC + " [e4m3 operands for QKV, O, W1||W3 and W2]",
        "value": S / (ms * 1e-3),
        "unit": UNIT, "n_gpus": 1, "steps": steps, "warmup": warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "e4m3 (QKV, O, W1||W3, W2) + bf16 (attention)",
        "data": "synthetic (seeded random-init weights and activations)",
        "config": {"workload": WORKLOADS[cfg], "S": S, "valid_rows": V},
        "tflops": tflops, "frac_of_bf16_burst_peak": tflops / peaks["bf16_tflops"],
        "clocks": clk.summary(),
        "qkv_w13_only": {"ms_per_step": ms_two, "value": S / (ms_two * 1e-3),
                         "tflops": block_flops(dims, V) / (ms_two * 1e-3) / 1e12},
    }
    layout.close()
    return line


FORWARD_WORKLOAD = ("full MiniMax-H3 transformer forward: fp32 patch projections (96 / 32 "
                    "channels), text projection (5120) and 2 refiner blocks, the 50-block stack "
                    "over the 16384-row padded layout (15872 valid rows, two timesteps), norm_out "
                    "and the fp32 video / audio heads")



def run_e4m3(args):
    print(json.dumps(e4m3_measure(args.steps, args.warmup, args.workload)))
    return 0


def run_ulysses(args):
    """--ulysses P: one rank's share of the sequence-parallel block on this GPU.
    Rank 0 of P runs its row chunk's norm + QKV (storing each head's rows into
    the owning rank's receive buffer), attention of its NH / P heads over every
    row (storing each row's output into the owning rank's buffer) and its
    chunk's O, norm and FFN. The receive buffers of all ranks live on this GPU,
    so the exchange stores land in local memory: the figure is one rank's
    compute, with the NVLink transfer time given beside it from the bytes each
    rank sends and the measured 770 GB/s per direction. The plain block on the
    same GPU is timed for comparison."""
    import types
    import torch
    from audio_generation_b200 import h3
    from audio_generation_b200.ulysses import UlyssesBlock

    P = args.ulysses
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    dims = FULL_DIMS
    d = h3.make_dims(dims)
    cfg = args.workload
    L = config_layout(cfg)
    S, V = L.S, L.n_valid
    if S % P or dims.heads % P or not 1 <= P <= 8:
        raise SystemExit("--ulysses P needs S % P == 0, heads % P == 0 and P <= 8")
    bits = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(
        torch.bfloat16)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
    w = block_weights(dims, cfg, 0)
    wd = types.SimpleNamespace(**{k: bits(getattr(w, k)) for k in ("w_qkv", "q_norm", "k_norm",
                                                                  "w_o", "w13", "w2")})
    wd.ada_table = f32(w.ada_table)
    pw = prologue_weights(dims, cfg)
    tws_b = h3.h3_timestep_workspace_size(d, L.n_t)
    tws = torch.empty(tws_b, dtype=torch.uint8, device=device)
    tmod = torch.empty((L.n_t, 6, dims.hidden), dtype=torch.float32, device=device)
    h3.h3_timestep_modulation(d, L.n_t, f32(L.timestep), f32(pw.w_t1), f32(pw.w_t2),
                              f32(pw.w_proj), tmod, tws, tws_b)
    del tws
    xb = activations(dims, cfg, S, 1)
    ranks = [UlyssesBlock(dims, L, r, P, device) for r in range(P)]
    Sr, NHl, D, H = S // P, dims.heads // P, dims.head_dim, dims.hidden
    peers = [h3.make_peers(r, *[[ranks[j].recv[i] for j in range(P)] for i in range(4)])
             for r in range(P)]
    xs = [bits(np.ascontiguousarray(xb[:, r * Sr:(r + 1) * Sr])) for r in range(P)]
    for r, rk in enumerate(ranks):  # every rank's q, k, v in place before rank 0's attention
        rk.pre_attention_to_heads(wd, tmod, xs[r], peers[r])
    x0 = xs[0].clone()
    stream = torch.cuda.current_stream(device)
    r0 = ranks[0]

    def rank0_step():
        xs[0].copy_(x0)
        r0.pre_attention_to_heads(wd, tmod, xs[0], peers[0])
        r0.attention_to_rows(peers[0])
        r0.post_attention(wd, tmod, r0.recv[3][None], xs[0])

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / args.steps

    ms_rank = timed(rank0_step)
    for rk in ranks:
        if h3.h3_layout_error(rk.full) != h3.H3_OK or h3.h3_layout_error(rk.chunk) != h3.H3_OK:
            raise RuntimeError("device error word set during the sequence-parallel run")
        rk.close()
    del ranks, peers, xs, r0
    torch.cuda.empty_cache()
    # the plain block on the same GPU
    layout = h3.h3_layout_prepare(d, S, L.n_t, f32(L.pos), i32(L.tags), i32(L.t_idx),
                                  i32(L.video_idx), i32(L.audio_idx), i32(L.text_idx))
    cw = h3.make_block_weights(wd.w_qkv, wd.q_norm, wd.k_norm, wd.w_o, wd.w13, wd.w2,
                               wd.ada_table)
    x = bits(xb)
    ws_b = h3.h3_workspace_size(d, 1, S)
    ws = torch.empty(ws_b, dtype=torch.uint8, device=device)
    ms_block = timed(lambda: h3.h3_block_forward(d, cw, layout, tmod, x, 1, ws, ws_b, stream))
    layout.close()
    # bytes one rank sends: q, k, v of its rows for the other ranks' heads, and
    # the attention output of the other ranks' rows for its heads
    out_bytes = 3 * Sr * (dims.heads - NHl) * D * 2 + (S - Sr) * NHl * D * 2
    line = {
        "metric": f"one rank's compute per block step, sequence-parallel over {P} ranks "
                  "(bf16, measured on 1xB200, exchange stores to local memory)",
        "value": ms_rank, "unit": "ms", "higher_is_better": False, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "dtype": "bf16",
        "data": "synthetic (seeded random-init weights and activations)",
        "config": {"workload": WORKLOADS[cfg], "S": S, "valid_rows": V, "ranks": P,
                   "rows_per_rank": Sr, "heads_per_rank": NHl},
        "single_gpu_block_ms": ms_block,
        "per_rank_share_of_block": ms_rank / ms_block,
        "exchange_bytes_sent_per_rank": out_bytes,
        "exchange_ms_at_770_GBps": out_bytes / 770e9 * 1e3,
        "note": "a P-GPU step is at least the per-rank compute; the exchange is stored by the "
                "producing kernels and overlaps them on NVLink, not measured here",
    }
    print(json.dumps(line))
    return 0

def run_forward(args):
    """--forward: one whole transformer forward (h3_forward) on one GPU, from
    latent rows to velocities. Prints one JSON line: forward time, valid rows/s
    and TFLOP/s over the algorithmic flops of the stack, the refiner (over the
    text rows) and the projections and heads."""
    import torch
    from audio_generation_b200 import h3
    from workloads import denoiser_inputs, denoiser_weights

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    dims = FULL_DIMS
    d, io = h3.make_dims(dims), h3.make_io_dims(dims)
    L = config_layout(STACK_CFG)
    S, V = L.S, L.n_valid
    nt_rows = len(L.text_idx)
    bits = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(
        torch.bfloat16)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)

    def dev_block(w):
        t = {k: bits(getattr(w, k)) for k in ("w_qkv", "q_norm", "k_norm", "w_o", "w13", "w2")}
        t["ada_table"] = f32(w.ada_table)
        return t, h3.make_block_weights(t["w_qkv"], t["q_norm"], t["k_norm"], t["w_o"], t["w13"],
                                        t["w2"], t["ada_table"])

    keep, blocks = [], []
    for i in range(STACK_BLOCKS):
        t, c = dev_block(block_weights(dims, STACK_CFG, i))
        keep.append(t)
        blocks.append(c)
    dw = denoiser_weights(dims, STACK_CFG)
    refiner = []
    for w in dw.refiner:
        t, c = dev_block(w)
        keep.append(t)
        refiner.append(c)
    iot = [f32(dw.w_patch_video), f32(dw.w_patch_audio), bits(dw.w_text), f32(dw.w_t1),
           f32(dw.w_t2), f32(dw.w_proj), f32(dw.w_out), f32(dw.out_table), f32(dw.w_head_video),
           f32(dw.w_head_audio)]
    iw = h3.make_io_weights(*iot)
    layout = h3.h3_layout_prepare(d, S, L.n_t, f32(L.pos), i32(L.tags), i32(L.t_idx),
                                  i32(L.video_idx), i32(L.audio_idx), i32(L.text_idx))
    video, audio, text = denoiser_inputs(dims, STACK_CFG, L)
    v_d, a_d, t_d, ts = f32(video), f32(audio), bits(text), f32(L.timestep)
    vo = torch.empty((1, len(L.video_idx), dims.video_channels), device=device)
    ao = torch.empty((1, len(L.audio_idx), dims.audio_in_channels), device=device)
    ws_b = h3.h3_forward_workspace_size(d, io, layout, 1)
    ws = torch.empty(ws_b, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def forward():
        h3.h3_forward(d, io, iw, refiner, blocks, layout, ts, 1, v_d, a_d, t_d, vo, ao, ws, ws_b,
                      stream)

    for _ in range(args.warmup):
        forward()
    torch.cuda.synchronize(device)
    gpu_id = torch.cuda.get_device_properties(device).uuid
    gpu_id = f"GPU-{gpu_id}" if not str(gpu_id).startswith("GPU-") else str(gpu_id)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id) as clk:
        time.sleep(0.3)
        e0.record(stream)
        for _ in range(args.steps):
            forward()
        e1.record(stream)
        torch.cuda.synchronize(device)
    if h3.h3_layout_error(layout) != h3.H3_OK:
        raise RuntimeError("device error word set during the forward run")
    ms = e0.elapsed_time(e1) / args.steps
    # core residual reuse: one forward that stores the stack's change, then
    # forwards that reuse it (the refiner and the 50 blocks skipped)
    core = torch.empty((1, V, dims.hidden), dtype=torch.float32, device=device)
    h3.h3_forward(d, io, iw, refiner, blocks, layout, ts, 1, v_d, a_d, t_d, vo, ao, ws, ws_b,
                  stream, core, h3.H3_CORE_STORE)
    for _ in range(args.warmup):
        h3.h3_forward(d, io, iw, refiner, blocks, layout, ts, 1, v_d, a_d, t_d, vo, ao, ws, ws_b,
                      stream, core, h3.H3_CORE_REUSE)
    torch.cuda.synchronize(device)
    e0.record(stream)
    for _ in range(args.steps):
        h3.h3_forward(d, io, iw, refiner, blocks, layout, ts, 1, v_d, a_d, t_d, vo, ao, ws, ws_b,
                      stream, core, h3.H3_CORE_REUSE)
    e1.record(stream)
    torch.cuda.synchronize(device)
    if h3.h3_layout_error(layout) != h3.H3_OK:
        raise RuntimeError("device error word set during the core-reuse run")
    ms_reuse = e0.elapsed_time(e1) / args.steps
    H = dims.hidden
    flops = (STACK_BLOCKS * block_flops(dims, V) + 2 * block_flops(dims, nt_rows)
             + 2.0 * nt_rows * dims.text_dim * H
             + 2.0 * 2 * H * (len(L.video_idx) * dims.video_channels
                              + len(L.audio_idx) * dims.audio_in_channels))
    peaks = load_peaks()
    tflops = flops / (ms * 1e-3) / 1e12
    line = {
        "metric": "valid packed rows/s per transformer forward (bf16 stack, 1xB200)",
        "value": V / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic (seeded random-init weights and latents)",
        "config": {"workload": FORWARD_WORKLOAD, "S": S, "valid_rows": V, "blocks": STACK_BLOCKS,
                   "refiner_blocks": len(refiner), "text_rows": nt_rows, "n_t": int(L.n_t)},
        "tflops": tflops, "frac_of_sustained_peak": tflops / peaks["bf16_tflops_sustained"],
        "frac_of_burst_peak": tflops / peaks["bf16_tflops"], "clocks": clk.summary(),
        "core_reuse": {"ms_per_step": ms_reuse,
                       "note": "H3_CORE_REUSE forward: projections, norm_out and heads over the "
                               "stored core residual (refiner and stack skipped)"},
    }
    print(json.dumps(line))
    layout.close()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", type=int, choices=sorted(WORKLOADS), default=DEFAULT_CFG,
                    help="single-block workload (4: 32768 rows; 3: 16384 padded; 2: 8192)")
    ap.add_argument("--ref-rows", type=int, default=256,
                    help="query rows per bounded oracle sample (one reference step)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-stack", action="store_true",
                    help="skip the 50-block stack measurement added to the block line")
    ap.add_argument("--no-masked", action="store_true",
                    help="skip the masked-attention measurement on the padded layout")
    ap.add_argument("--ulysses", type=int, default=0,
                    help="time one rank's share of the sequence-parallel block over this many ranks")
    ap.add_argument("--reduced", action="store_true",
                    help="with --stack: also time the token-reduced stack")
    ap.add_argument("--stack", action="store_true",
                    help="time the 50-block stack forward instead (one GPU, own JSON line)")
    ap.add_argument("--attention-only", action="store_true",
                    help="time the attention kernel alone on the workload (own JSON line)")
    ap.add_argument("--e4m3", action="store_true",
                    help="time the block with e4m3 QKV and W1||W3 operands instead (own JSON line)")
    ap.add_argument("--forward", action="store_true",
                    help="time the whole transformer forward instead (one GPU, own JSON line)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.ulysses:
        return run_ulysses(args)
    if args.stack:
        return run_stack(args)
    if args.forward:
        return run_forward(args)
    if args.e4m3:
        return run_e4m3(args)
    if args.attention_only:
        return run_attention_only(args)
    return run_gpu(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
