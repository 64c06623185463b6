"""Benchmark of the VDN hybrid video-video attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 768p-bf16]
                    [--entry hybrid|window|window-fp8|vda|vda-decay|hybrid-decay|joint|joint-window]

A step is one vdn_hybrid_attn_fwd call (window softmax + VDA scans + readout,
norm, gates) over one 768p-like layer input (B=1, H=40, d=128, F=36 frames of
48 x 84 tokens, chunks of 5, 512 text tokens) resident in HBM. Inputs are
larger than L2 (each video tensor is 1.49 GB), so L2 is not flushed.

For N > 1 (launched by torchrun) every rank runs its own independent layer
input (weak scaling, no collective in the data path); the timed region is
bracketed by a barrier and device synchronisation on every rank and the
reported time is the maximum over ranks.

--entry selects the public entry point that forms the step: the hybrid
forward (default, the headline), or the softmax branch or the linear branch
alone (vdn_window_softmax_fwd / vdn_vda_scan_fwd), for per-branch numbers and
for profiling one kernel family at a time, or the KDA-decayed forms
(vdn_vda_scan_fwd_decay / vdn_hybrid_attn_fwd_decay, alpha in (0.8, 1]), or
the joint text-video-audio layer (vdn_joint_attn_fwd / vdn_joint_softmax_fwd:
audio keys for every video query, dense text and audio query rows; the audio
length that goes with the clip, 203 tokens at 768p), or the softmax branch with
float8 e4m3 operands (vdn_window_softmax_fwd_fp8).

Printed on rank 0: one JSON line with the throughput (video tokens/s over all
ranks), the roofline of the dominant kernel (window softmax, tensor-core bound),
the roofline of the linear branch (vdn_vda_scan_fwd, HBM-bound),
the end-to-end figure through the public call with host buffers, the CPU
oracle baseline on a bounded sample, and the SM clocks seen during timing.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "hybrid-attn fwd video tokens/s on 1 B200 (768p-like); % of TC/HBM roofline"
UNIT = "video tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------ algorithmic work

def window_pairs(lay) -> int:
    """Allowed (query, key) pairs of one (b, h): every query token of frame f sees
    the tokens of its window + anchor frames and all text tokens."""
    F, N, T, c = lay.F, lay.N, lay.T, lay.c
    total = 0
    for f in range(F):
        if f == 0 or f == F - 1:
            frames = F
        else:
            j = f // c
            lo, hi = max(0, c * (j - 1)), min(F - 1, c * (j + 2) - 1)
            frames = hi - lo + 1 + (1 if lo > 0 else 0) + (1 if hi < F - 1 else 0)
        total += N * (frames * N + T)
    return total


def window_flops(lay) -> float:
    """4 d flops per allowed pair (q.k and p.v), all heads and batches."""
    return 4.0 * lay.d * window_pairs(lay) * lay.H * lay.B


def joint_flops(lay, A) -> float:
    """Window flops of a joint layer: every video query also sees the A audio
    keys, and the T text + A audio query rows see every video, text and audio
    key (4 d flops per pair)."""
    extra = lay.L * A + (lay.T + A) * (lay.L + lay.T + A)
    return window_flops(lay) + 4.0 * lay.d * extra * lay.H * lay.B


def launches_per_step(lay, dtype) -> int:
    """Kernels of one vdn_hybrid_attn_fwd call: the frame Gram (bf16: with the
    inverse (I + A_f)^-1 in its epilogue; fp32: a separate inverse kernel), the
    scan, the zero-fill of unused chunk entries, the window softmax (float32
    o_soft) and the readout finishing the output (o_lin, RMSNorm, gates)."""
    return 5 if dtype == "bf16" else 6


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self):
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self, gpu_indices):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                idx = int(p[0])
            except ValueError:
                continue
            if gpu_indices is not None and idx not in gpu_indices:
                continue
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
            except ValueError:
                continue
            for n, val in zip(names, p[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [x for x in sm if x > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def window_kernel_traffic(lay):
    """Per-launch DRAM bytes of the window-softmax kernel from the committed ncu
    summary, scaled to this workload; None when the summary is missing or was
    taken on a different kernel source."""
    p = os.path.join(ROOT, "profiles", "window_tc_traffic.txt")
    src = os.path.join(ROOT, "linear_attention_video_block_b200", "csrc", "window_tc.cu")
    if not os.path.exists(p) or not os.path.exists(src):
        return None
    kv = {}
    for line in open(p):
        if "=" in line and not line.startswith("#"):
            a, b = line.split("=", 1)
            kv[a.strip()] = b.strip()
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if kv.get("source_sha256_16") != digest:
        return None
    try:
        bytes_per_pair = float(kv["dram_bytes_per_allowed_pair_head"])
    except (KeyError, ValueError):
        return None
    return bytes_per_pair * window_pairs(lay) * lay.H * lay.B


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own independent layer input (weak scaling)."""
    return seed + rank


def max_over_ranks(values, world: int, device="cpu"):
    """Element-wise maximum of per-rank timings over all ranks (the job's time is
    that of its slowest rank). A no-op for a single rank."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(tokens_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job video tokens/s: all ranks' tokens over the slowest rank's time."""
    return tokens_per_rank * world / (max_ms * 1e-3)


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(lay, dtype, seed, rows_per_frame):
    """Times the float64 oracle on a bounded sample of the workload: one head
    drawn with the workload's recipe, the whole linear branch of that head, and
    the softmax branch, norm and gates on `rows_per_frame` query rows of every
    frame. Returns (extrapolated video tokens/s for the whole workload, seconds,
    description)."""
    import numpy as np
    from linear_attention_video_block_b200.synth import Layout, make_inputs
    from oracle import vdn_oracle as O

    one = Layout(B=1, F=lay.F, N=lay.N, T=lay.T, c=lay.c, H=1, d=lay.d)
    inp = make_inputs(one, dtype, seed)
    a = {k: v.double().numpy() for k, v in inp.items()}
    rng = np.random.default_rng(0)
    rows = np.sort(np.concatenate([f * lay.N + rng.choice(lay.N, rows_per_frame, replace=False)
                                   for f in range(lay.F)]))
    t0 = time.perf_counter()
    o_lin = O.linear_branch(a["q"], a["k"], a["v"], a["k_text"], a["v_text"], a["beta"],
                            a["beta_text"], lay.F, lay.N, lay.c)
    t1 = time.perf_counter()
    o_soft = O.softmax_branch(a["q"], a["k"], a["v"], a["k_text"], a["v_text"], lay.F, lay.N,
                              lay.c, rows=rows)
    O.combine(o_soft[:, rows], o_lin[:, rows], a["g_s"][:, rows], a["g_l"][:, rows])
    t2 = time.perf_counter()
    per_head = (t1 - t0) + (t2 - t1) * (lay.L / len(rows))
    est = per_head * lay.H * lay.B
    desc = (f"1 of {lay.H} heads drawn with the same recipe; linear branch in full, softmax + "
            f"gates on {rows_per_frame} query rows per frame ({len(rows)} of {lay.L}); "
            f"extrapolated linearly to all rows and heads")
    return lay.L * lay.B / est, t2 - t0, desc


# ---------------------------------------------------------------- arms

def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores (rank 0 only)."""
    from linear_attention_video_block_b200.synth import WORKLOADS
    if rank != 0:
        return
    lay, dtype, seed = WORKLOADS[args.workload]
    rpf = args.ref_rows
    for _ in range(args.warmup):
        oracle_sample(lay, dtype, seed, rpf)
    vals, secs = [], []
    desc = ""
    for _ in range(args.steps):
        v, s, desc = oracle_sample(lay, dtype, seed, rpf)
        vals.append(v)
        secs.append(s)
    value = statistics.median(vals)
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * lay.L * lay.B / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(args.workload, lay),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(name, lay):
    return {"workload": name, "B": lay.B, "F": lay.F, "N": lay.N, "T": lay.T, "c": lay.c,
            "H": lay.H, "d": lay.d, "video_tokens": lay.L * lay.B,
            "l2": "inputs larger than L2 (1.49 GB per video tensor); no flush",
            "parallelism": "independent problem per GPU (weak scaling)"}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from linear_attention_video_block_b200 import vdn
    from linear_attention_video_block_b200.synth import WORKLOADS, make_inputs

    lay, dtype, seed = WORKLOADS[args.workload]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    inp = make_inputs(lay, dtype, rank_seed(seed, rank), device=str(dev))
    ws = torch.empty(vdn.workspace_bytes(lay, inp["q"].dtype), dtype=torch.uint8, device=dev)
    out = torch.empty_like(inp["q"])
    stream = torch.cuda.current_stream(dev)

    def step():
        vdn.hybrid_attn_fwd(lay, inp["q"], inp["k"], inp["v"], inp["k_text"], inp["v_text"],
                            inp["beta"], inp["beta_text"], inp["g_s"], inp["g_l"], out=out,
                            workspace=ws)

    def barrier():
        if world > 1:
            dist.barrier()

    # The linear branch alone (vdn_vda_scan_fwd: Gram, inverse, scans, zero
    # fill, readout), HBM-bound. Timed first, before any window-kernel launch:
    # a second of the power-capped window kernel leaves the clocks low for the
    # launches that follow, and this is the branch's own speed.
    o_lin = torch.empty_like(inp["q"])

    def vda_call():
        vdn.vda_scan_fwd(lay, inp["q"], inp["k"], inp["v"], inp["k_text"], inp["v_text"], inp["beta"],
                         inp["beta_text"], o_lin=o_lin, workspace=ws)

    vda_launches = max(args.steps, 20)
    for _ in range(max(args.warmup, 3)):
        vda_call()
    torch.cuda.synchronize(dev)
    v0 = torch.cuda.Event(enable_timing=True)
    v1 = torch.cuda.Event(enable_timing=True)
    v0.record(stream)
    for _ in range(vda_launches):
        vda_call()
    v1.record(stream)
    torch.cuda.synchronize(dev)
    vda_ms = v0.elapsed_time(v1) / vda_launches
    del o_lin

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert vdn.device_status() == 0, "device status set during warm-up"

    clocks = ClockSampler()
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = e0.elapsed_time(e1) / args.steps

    # The dominant kernel alone: the window-softmax launch of the same
    # configuration, timed over the same number of launches.
    o_soft = torch.empty_like(inp["q"])
    for _ in range(2):
        vdn.window_softmax_fwd(lay, inp["q"], inp["k"], inp["v"], inp["k_text"], inp["v_text"],
                               o_soft=o_soft)
    torch.cuda.synchronize(dev)
    w0 = torch.cuda.Event(enable_timing=True)
    w1 = torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    for _ in range(args.steps):
        vdn.window_softmax_fwd(lay, inp["q"], inp["k"], inp["v"], inp["k_text"], inp["v_text"],
                               o_soft=o_soft)
    w1.record(stream)
    torch.cuda.synchronize(dev)
    win_ms = w0.elapsed_time(w1) / args.steps

    clk = clocks.stop(None) if rank == 0 else None

    # End to end through the public call with pinned host buffers: every step
    # copies the inputs in and the output back.
    host = {k: v.cpu().pin_memory() for k, v in inp.items()}
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size()

    # the input copies and the video tensors of the device leg are released
    # first: the host call keeps its own two chunk buffers on the device
    del inp, out, o_soft, ws
    torch.cuda.empty_cache()
    ws_h = torch.empty(vdn.host_workspace_bytes(lay, host["q"].dtype), dtype=torch.uint8, device=dev)

    def e2e_step():
        vdn.hybrid_attn_fwd_host(lay, host["q"], host["k"], host["v"], host["k_text"], host["v_text"],
                                 host["beta"], host["beta_text"], host["g_s"], host["g_l"], out=out_h,
                                 workspace=ws_h, device=str(dev))

    e2e_step()
    torch.cuda.synchronize(dev)
    e2e_steps = max(1, min(args.steps, 5))
    barrier()
    x0 = torch.cuda.Event(enable_timing=True)
    x1 = torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    x1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = x0.elapsed_time(x1) / e2e_steps
    assert vdn.device_status() == 0, "device status set during timing"

    ms, win_ms, vda_ms, e2e_ms = max_over_ranks([ms, win_ms, vda_ms, e2e_ms], world, device=dev)
    if rank != 0:
        return
    tokens = lay.L * lay.B * world
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    flops = window_flops(lay)
    achieved = flops / (win_ms * 1e-3) / 1e12
    traffic = window_kernel_traffic(lay)
    cpu_val, cpu_s, cpu_desc = oracle_sample(lay, dtype, seed, args.ref_rows)
    line = {
        "impl": "ours", "metric": METRIC, "value": job_throughput(lay.L * lay.B, world, ms), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
        "data": "synthetic (seeded: q, v, gates ~ N(0,1); k ~ N(0,1) L2-normalised; "
                "beta = sigmoid(N(0,1)))",
        "config": config_of(args.workload, lay),
        "roofline": {"bound": "tensor", "kernel": "window softmax (tcgen05)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_kind} bf16 dense (burst)",
                     "flops_per_launch": flops, "launch_ms": win_ms,
                     "share_of_step": win_ms / ms,
                     # the same against the matmul peak held for seconds under the
                     # power cap (the kernel runs for seconds in this measurement)
                     "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak))},
        "roofline_vda": dict(vda_roofline(lay, vda_ms, peaks, peak_kind), launches=vda_launches,
                             timed="alone, before the first window-kernel launch"),
        "cpu_baseline": {"value": cpu_val, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                         "sample": cpu_desc, "seconds": cpu_s},
        "e2e": {"value": job_throughput(lay.L * lay.B, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps},
        "clocks": clk,
        "gpu_launches": launches_per_step(lay, dtype) * args.steps * world,
        "when": datetime.datetime.now(datetime.timezone.utc).isoformat(timespec="seconds"),
    }
    print(json.dumps(line), flush=True)


def vda_bytes(lay) -> float:
    """Algorithmic HBM bytes of vdn_vda_scan_fwd: k, v and beta of the scanned
    frames and the text, q read and o_lin written once, the chunk table."""
    from linear_attention_video_block_b200.synth import Layout  # noqa: F401
    F, N, T, c, H, d, B = lay.F, lay.N, lay.T, lay.c, lay.H, lay.d, lay.B
    J = -(-F // c)
    fwd_max, rev_min = 0, F - 1
    for j in range(J):
        f0, f1 = max(j * c, 1), min((j + 1) * c - 1, F - 2)
        if f1 < f0:
            continue
        lo, hi = max(0, c * (j - 1)), min(F - 1, c * (j + 2) - 1)
        fwd_max = max(fwd_max, lo - 1 if lo - 1 >= 1 else 0)
        rev_min = min(rev_min, hi + 1 if hi + 1 <= F - 2 else F - 1)
    frames = set(range(1, fwd_max + 1)) | set(range(rev_min, F - 1))
    tok = len(frames) * N + T
    per_bh = tok * (2 * d * 2 + 4) + 2 * F * N * d * 2 + 2 * J * d * d * 4
    return float(per_bh * H * B)


def vda_roofline(lay, ms, peaks, peak_kind):
    """Roofline object of the linear-branch entry (HBM-bound): its algorithmic
    bytes per launch (vda_bytes) over the measured launch time, against the
    measured HBM copy bandwidth."""
    peak = float(peaks["hbm_gbs"])
    nbytes = vda_bytes(lay)
    achieved = nbytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "linear branch (vdn_vda_scan_fwd: gram, inverse, scans, "
                                      "readout)",
            "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": None, "peak_source": f"{peak_kind} HBM copy bandwidth",
            "bytes_per_launch": nbytes, "launch_ms": ms}


def decay_bytes(lay) -> float:
    """Extra algorithmic bytes of the decayed scans: alpha [B, F, H, d] fp32 of
    the non-boundary frames, read once."""
    return float(lay.B * max(lay.F - 2, 0) * lay.H * lay.d * 4)


def run_entry(args, rank, world, local_rank):
    """One entry point as the step (no e2e / CPU baseline legs): a branch alone,
    or the _decay forms of the linear branch and the hybrid forward."""
    import torch
    from linear_attention_video_block_b200 import vdn
    from linear_attention_video_block_b200.synth import (WORKLOADS, audio_tokens, make_context,
                                                         make_decay, make_inputs, quantize_e4m3)

    lay, dtype, seed = WORKLOADS[args.workload]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    inp = make_inputs(lay, dtype, rank_seed(seed, rank), device=str(dev))
    alpha = make_decay(lay, rank_seed(seed, rank) + 1, device=str(dev))
    out = torch.empty_like(inp["q"])
    ws = torch.empty(vdn.workspace_bytes(lay, inp["q"].dtype), dtype=torch.uint8, device=dev)
    A = audio_tokens(lay.F)
    cx = make_context(lay, A, dtype, rank_seed(seed, rank) + 7, device=str(dev)) \
        if args.entry.startswith("joint") else None
    if args.entry == "window":
        def step():
            vdn.window_softmax_fwd(lay, inp["q"], inp["k"], inp["v"], inp["k_text"], inp["v_text"],
                                   o_soft=out)
    elif args.entry == "window-fp8":
        (q8,), sq = quantize_e4m3(inp["q"])
        (k8, kt8), sk = quantize_e4m3(inp["k"], inp["k_text"])
        (v8, vt8), sv = quantize_e4m3(inp["v"], inp["v_text"])

        def step():
            vdn.window_softmax_fwd_fp8(lay, q8, k8, v8, kt8, vt8, sq, sk, sv, o_soft=out)
    elif args.entry == "joint":
        o_text, o_audio = torch.empty_like(cx["q_text"]), torch.empty_like(cx["q_audio"])

        def step():
            vdn.joint_attn_fwd(lay, inp["q"], inp["k"], inp["v"], inp["k_text"], inp["v_text"],
                               inp["beta"], inp["beta_text"], inp["g_s"], inp["g_l"],
                               k_audio=cx["k_audio"], v_audio=cx["v_audio"], q_text=cx["q_text"],
                               q_audio=cx["q_audio"], out=out, o_text=o_text, o_audio=o_audio,
                               workspace=ws)
    elif args.entry == "joint-window":
        o_text, o_audio = torch.empty_like(cx["q_text"]), torch.empty_like(cx["q_audio"])

        def step():
            vdn.joint_softmax_fwd(lay, inp["q"], inp["k"], inp["v"], inp["k_text"], inp["v_text"],
                                  k_audio=cx["k_audio"], v_audio=cx["v_audio"], q_text=cx["q_text"],
                                  q_audio=cx["q_audio"], o_soft=out, o_text=o_text, o_audio=o_audio)
    elif args.entry == "hybrid-decay":
        def step():
            vdn.hybrid_attn_fwd(lay, inp["q"], inp["k"], inp["v"], inp["k_text"], inp["v_text"],
                                inp["beta"], inp["beta_text"], inp["g_s"], inp["g_l"], out=out,
                                workspace=ws, alpha=alpha)
    else:
        a = alpha if args.entry == "vda-decay" else None

        def step():
            vdn.vda_scan_fwd(lay, inp["q"], inp["k"], inp["v"], inp["k_text"], inp["v_text"],
                             inp["beta"], inp["beta_text"], o_lin=out, workspace=ws, alpha=a)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    assert vdn.device_status() == 0
    ms = e0.elapsed_time(e1) / args.steps
    if rank != 0:
        return
    peaks, kind = load_peaks()
    if args.entry == "window":
        work, unit, peak = window_flops(lay) / 1e12, "TFLOP/s", float(peaks["bf16_tflops"])
        bound = "tensor"
    elif args.entry == "joint-window":
        work, unit, peak = joint_flops(lay, A) / 1e12, "TFLOP/s", float(peaks["bf16_tflops"])
        bound = "tensor"
    elif args.entry == "window-fp8":
        # e4m3 dense peak: the measured bf16 peak times the nominal fp8 / bf16 ratio (2)
        work, unit, peak = window_flops(lay) / 1e12, "TFLOP/s", 2.0 * float(peaks["bf16_tflops"])
        bound = "tensor"
        kind = f"{kind} bf16 x 2 (nominal e4m3 / bf16 ratio)"
    elif args.entry in ("hybrid-decay", "joint"):
        work, unit, peak, bound = None, None, None, None
    else:
        extra = decay_bytes(lay) if args.entry == "vda-decay" else 0.0
        work, unit, peak = (vda_bytes(lay) + extra) / 1e9, "GB/s", float(peaks["hbm_gbs"])
        bound = "hbm"
    roof = None
    if work is not None:
        ach = work / (ms * 1e-3)
        roof = {"bound": bound, "achieved": ach, "peak": peak, "unit": unit,
                "frac": ach / peak, "peak_source": kind}
    print(json.dumps({
        "impl": "ours", "entry": args.entry, "metric": f"{args.entry} fwd video tokens/s",
        "value": lay.L * lay.B / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "dtype": "e4m3" if args.entry == "window-fp8" else dtype,
        "config": dict(config_of(args.workload, lay),
                       **({"audio_tokens": A, "context_query_rows": lay.T + A}
                          if args.entry.startswith("joint") else {})),
        "roofline": roof,
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="768p-bf16")
    ap.add_argument("--entry", choices=["hybrid", "window", "window-fp8", "vda", "vda-decay",
                                        "hybrid-decay", "joint", "joint-window"], default="hybrid")
    ap.add_argument("--ref-rows", type=int, default=96,
                    help="query rows per frame in the oracle's bounded sample")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.entry == "hybrid":
            run_ours(args, rank, world, local_rank)
        else:
            run_entry(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
