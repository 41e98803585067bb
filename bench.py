#!/usr/bin/env python
"""Benchmark of the LittleBit layer forward on B200; prints ONE JSON line.

Default workload (one "step" = one forward over a stack of layers, batch 1):
the Llama-2-70B MLP stack at 0.1 BPW, single path s = 620 (8192 -> 28672 gate
and up, 28672 -> 8192 down per model layer), 80 distinct model layers (own
signs, scales, input and output; 722 MB of packed weights, 5.7x the L2 cache),
so that every step streams its weights from HBM.  The metric is microseconds
per model layer; the roofline object reports the dominant kernel's achieved
HBM GB/s.  The residual variant of the same stack, the Llama-2-7B full linear
stack and the prefill stack are reported as secondary figures.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (the only other place that runs the oracle).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode µs/layer & % HBM roofline at batch 1; prefill TFLOP/s & % tensor peak"
FALLBACK_HBM_GBS = 6650.0

# (d_in, d_out, s, residual) per matrix of one model layer
WORKLOADS = {
    "7b_attn_0.1bpw_residual": {
        "desc": "Llama-2-7B attention projection 4096x4096, 0.1 BPW residual (s=86 x 2 paths)",
        "mats": [(4096, 4096, 86, True)],
    },
    "7b_attn_0.1bpw_single": {
        "desc": "Llama-2-7B attention projection 4096x4096, 0.1 BPW single path (s=188)",
        "mats": [(4096, 4096, 188, False)],
    },
    "70b_mlp_0.1bpw_single": {
        "desc": "Llama-2-70B MLP layer (8192->28672 gate, up; 28672->8192 down), 0.1 BPW single path s=620",
        "mats": [(8192, 28672, 620, False), (8192, 28672, 620, False), (28672, 8192, 620, False)],
        "model_layers": 80,
        "x_groups": [0, 0, 1],   # gate and up read the MLP's input
    },
    "70b_mlp_0.1bpw_residual": {
        "desc": "Llama-2-70B MLP layer, 0.1 BPW residual s=302 x 2 paths",
        "mats": [(8192, 28672, 302, True), (8192, 28672, 302, True), (28672, 8192, 302, True)],
        "model_layers": 80,
        "x_groups": [0, 0, 1],
    },
    "7b_layer_0.1bpw_residual": {
        "desc": "Llama-2-7B layer (4x 4096^2 s=86; 2x 4096->11008 and 11008->4096 s=133), 0.1 BPW residual",
        "mats": [(4096, 4096, 86, True)] * 4 + [(4096, 11008, 133, True)] * 2 + [(11008, 4096, 133, True)],
        "model_layers": 32,
        # q, k, v read the block's normalised input; gate and up read the MLP's
        "x_groups": [0, 0, 0, 1, 2, 2, 3],
    },
}
DEFAULT_WORKLOAD = "70b_mlp_0.1bpw_single"


def algorithmic_bytes(d_in, d_out, s, residual, batch):
    """Bytes the method must move for one matrix (packed bits at exactly s(a+b)
    bits per path, fp16 scales, fp16 input and output)."""
    paths = 2 if residual else 1
    per_path = s * (d_in + d_out) / 8 + 2 * (d_in + d_out + s)
    return paths * per_path + 2 * batch * (d_in + d_out)


KERNELS = ("quantise", "latent_pass", "finalize", "output_pass")


def kernel_bytes(d_in, d_out, s, residual, batch):
    """Algorithmic bytes split by decode kernel (they sum to algorithmic_bytes):
    quantise (g per path, x), latent pass (V bits), finalize (l), output pass
    (U bits, h, y)."""
    paths = 2 if residual else 1
    return {"quantise": paths * 2 * d_in + 2 * batch * d_in,
            "latent_pass": paths * s * d_in / 8,
            "finalize": paths * 2 * s,
            "output_pass": paths * (s * d_out / 8 + 2 * d_out) + 2 * batch * d_out}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return float(pk.get("hbm_gbs", FALLBACK_HBM_GBS)), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples while the GPU works."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,utilization.gpu,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        with open(self.tmp.name) as f:
            rows = [ln.strip().split(", ") for ln in f if ln.strip()]
        os.unlink(self.tmp.name)
        samples = []
        for r in rows:
            try:
                samples.append({"sm": float(r[1]), "max": float(r[2]), "util": float(r[3]),
                                "hw": r[6].strip(), "hwt": r[7].strip(), "swt": r[8].strip(), "pcap": r[9].strip()})
            except (ValueError, IndexError):
                continue
        if not samples:
            return None
        load = [s for s in samples if s["util"] > 0] or samples
        reasons = set()
        for s in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("pcap", "sw_power_cap")):
                if s[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s["sm"] for s in load), "sm_max_mhz": max(s["max"] for s in load),
                "reasons": sorted(reasons), "samples": len(load)}


def traffic_record(kernel: str, workload: str, model_layers: int):
    """dram bytes per launch of `kernel` from the committed ncu summary (bytes
    per model layer x the model layers of this launch), if it was taken on the
    current kernel source."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    src = os.path.join(ROOT, "latent_binary_factorization_b200", "csrc", "decode.cu")
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()[:16]
    r = rec.get(workload, {}).get(kernel)
    if not r or r.get("decode_cu_sha256_16") != digest:
        return None
    return int(r["dram_bytes_per_model_layer"] * model_layers)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def build_stack(mats, n_rep, batch, seed, device, x_groups=None):
    """n_rep model layers of distinct random layers; within a model layer the
    matrices of one x group read the same input tensor."""
    import torch
    from latent_binary_factorization_b200 import layers as lbl, littlebit as lb
    gen = torch.Generator(device=device).manual_seed(seed)
    groups = x_groups or list(range(len(mats)))
    Ls = []
    for _ in range(n_rep):
        for (a, b, s, r) in mats:
            Ls.append(lbl.random_layer(a, b, s, r, gen, device=device)[0])
    # one input per (model layer, group), back to back in x_all
    first = {}
    for k, g in enumerate(groups):
        first.setdefault(g, k)
    per_layer_x = sum(mats[k][0] for k in first.values())
    x_all = torch.randn(n_rep * per_layer_x * batch, generator=gen, device=device).half()
    y_all = torch.empty(sum(L.d_out for L in Ls) * batch, dtype=torch.float16, device=device)
    xs, ys, xo, yo = [], [], 0, 0
    for rep in range(n_rep):
        gx = {}
        for k, g in enumerate(groups):
            if g not in gx:
                a = mats[k][0]
                gx[g] = x_all[xo:xo + batch * a].view(batch, a)
                xo += batch * a
            xs.append(gx[g])
    for L in Ls:
        ys.append(y_all[yo:yo + batch * L.d_out].view(batch, L.d_out))
        yo += batch * L.d_out
    return lb.Stack(Ls, xs, ys), Ls, x_all, y_all


def shared_x_bytes(mats, x_groups, batch):
    """Input bytes not read again because matrices of a model layer share
    their x (one read per group instead of one per matrix)."""
    if not x_groups:
        return 0
    seen, saved = set(), 0
    for (a, _, _, _), g in zip(mats, x_groups):
        if g in seen:
            saved += 2 * batch * a
        seen.add(g)
    return saved


def layer_bytes(name, batch):
    """Algorithmic bytes of one model layer of a workload (shared inputs read once)."""
    wl = WORKLOADS[name]
    return (sum(algorithmic_bytes(*m, batch) for m in wl["mats"])
            - shared_x_bytes(wl["mats"], wl.get("x_groups"), batch))


def stack_reps_for_l2(mats, batch, l2_bytes, factor=4.0, model_layers=1):
    """Model layers per step: the model's own layer count, or more distinct
    copies if needed for the packed bytes to reach `factor` x L2."""
    per = sum(algorithmic_bytes(*m, batch) for m in mats)
    return max(1, model_layers, math.ceil(factor * l2_bytes / per))


def max_over_ranks(values, device):
    """Each value's maximum over all ranks of the default process group (a
    no-op with one process): device times of a multi-rank step are the
    slowest rank's."""
    import torch
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_us_per_layer(ms_per_step, layers_per_rank, world):
    """Whole-job figure: every rank runs its own stack of `layers_per_rank`
    layers per step (weak scaling), so one step processes layers_per_rank *
    world layers in the slowest rank's step time."""
    return 1e3 * ms_per_step / (layers_per_rank * world)


def time_device(stack, steps, warmup, dist):
    """K device-timed steps (CUDA events on the launching stream, nothing else
    recorded in between), then K more steps for each decode kernel's share,
    from events the library records after the first three of its four
    launches."""
    import torch
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        stack()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(steps):
        stack()
    t1.record(stream)
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    total_ms = t0.elapsed_time(t1)
    # per-kernel split (separate pass: the extra event records add small gaps)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for k in range(steps):
        ev[k][0].record(stream)
        # torch only times events it recorded itself; an event keeps its latest
        # record, so record the three inner ones here and let the library
        # re-record them after its quantise, latent and finalize launches
        for e in ev[k][1:4]:
            e.record(stream)
        stack(events=ev[k][1:4])
        ev[k][4].record(stream)
    torch.cuda.synchronize()
    per = {name: sum(e[i].elapsed_time(e[i + 1]) for e in ev) / steps for i, name in enumerate(KERNELS)}
    return total_ms, per


def measure_mixed(name, batch, steps, warmup, device, dist, l2, seed=4321):
    """A batch between the decode and prefill ranges (fp16): the leading
    multiple of 128 rows run on the prefill path and the rest on the decode
    path in groups of at most 16 rows, each group streaming the weights again.
    Whole-step time only (the per-kernel event split is a decode-only view)."""
    import torch
    mats = WORKLOADS[name]["mats"]
    reps = stack_reps_for_l2(mats, batch, l2)
    stack, Ls, x_all, y_all = build_stack(mats, reps, batch, seed, device)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        stack()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(steps):
        stack()
    t1.record(stream)
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    ms = max_over_ranks([t0.elapsed_time(t1) / steps], device)[0]
    alg = sum(algorithmic_bytes(*m, batch) for m in mats) * reps
    prefill_rows = batch // 128 * 128
    res = {"workload": name, "desc": WORKLOADS[name]["desc"], "batch": batch, "layers_per_step": len(Ls),
           "prefill_rows": prefill_rows, "decode_groups": -(-(batch - prefill_rows) // 16),
           "ms_per_step": ms, "us_per_matrix": 1e3 * ms / len(Ls),
           "us_per_matrix_row": 1e3 * ms / len(Ls) / batch,
           "step_gbs_algorithmic": alg / (ms * 1e-3) / 1e9}
    del stack, x_all, y_all
    torch.cuda.empty_cache()
    return res


def measure_latency(device, reps=200, seed=99):
    """Latency view: one Llama-2-7B attention projection (4096x4096, 0.1 BPW
    residual, s = 86 x 2) at batch 1 per call, its 0.1 MB of weights staying
    in L2 between calls.  Eager: back-to-back forward calls (host work and four
    launches each).  Graph: the same call captured once into a CUDA graph and
    replayed.  CUDA events on the stream, microseconds per call."""
    import torch
    from latent_binary_factorization_b200 import layers as lbl, littlebit as lb
    gen = torch.Generator(device=device).manual_seed(seed)
    L = lbl.random_layer(4096, 4096, 86, True, gen, device=device)[0]
    x = torch.randn(1, 4096, generator=gen, device=device).half()
    y = torch.empty(1, 4096, dtype=torch.float16, device=device)
    stack = lb.Stack([L], [x], [y])
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))
    out = {}
    with torch.cuda.stream(side):
        for _ in range(10):
            stack()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(side)
        for _ in range(reps):
            stack()
        e1.record(side)
        torch.cuda.synchronize(device)
        out["eager_us"] = round(1e3 * e0.elapsed_time(e1) / reps, 3)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        stack()
    with torch.cuda.stream(side):
        for _ in range(10):
            g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(side)
        for _ in range(reps):
            g.replay()
        e1.record(side)
        torch.cuda.synchronize(device)
        out["graph_us"] = round(1e3 * e0.elapsed_time(e1) / reps, 3)
    del g
    out["workload"] = "one Llama-2-7B attention projection 4096x4096, 0.1 BPW residual (s=86 x 2), batch 1, per call"
    return out


def time_e2e(stack, x_all, y_all, steps, warmup, n_chunks):
    """Same forward through the public host-buffer API: every step copies all
    layers' inputs in from pinned host memory, runs the stack and copies every
    output back (littlebit_linear_forward_many_host, in n_chunks overlapped
    groups of layers)."""
    import torch
    from latent_binary_factorization_b200 import littlebit as lb
    stream = torch.cuda.current_stream()
    hs = lb.HostStack(stack.layers, stack.batch, x_all.dtype)
    # the host call takes every layer's input back to back (a shared input is
    # copied once per layer that reads it)
    x_host = torch.cat([x.reshape(-1) for x in stack.xs]).cpu()
    xh = torch.empty(x_host.numel(), dtype=x_all.dtype, pin_memory=True)
    xh.copy_(x_host)
    yh = torch.empty(y_all.numel(), dtype=y_all.dtype, pin_memory=True)

    def step():
        hs(xh, yh, n_chunks=n_chunks, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1), xh.numel() * xh.element_size(), y_all.numel() * y_all.element_size()


def measure_workload(name, batch, steps, warmup, device, dist, world, l2, seed=1234, l2_factor=4.0):
    mats = WORKLOADS[name]["mats"]
    x_groups = WORKLOADS[name].get("x_groups")
    model_layers = WORKLOADS[name].get("model_layers", 1) if l2_factor >= 4.0 else 1
    reps = stack_reps_for_l2(mats, batch, l2, l2_factor, model_layers)
    stack, Ls, x_all, y_all = build_stack(mats, reps, batch, seed, device, x_groups)
    n_layers = len(Ls)
    total_ms, per_ms = time_device(stack, steps, warmup, dist)
    red = max_over_ranks([total_ms] + [per_ms[k] for k in KERNELS], device)
    total_ms, per_ms = red[0], dict(zip(KERNELS, red[1:]))
    alg = layer_bytes(name, batch) * reps
    kb = {k: sum(kernel_bytes(*m, batch)[k] for m in mats) * reps for k in KERNELS}
    kb["quantise"] -= shared_x_bytes(mats, x_groups, batch) * reps
    ms_step = total_ms / steps
    res = {
        "workload": name, "desc": WORKLOADS[name]["desc"], "batch": batch, "layers_per_step": n_layers,
        "shared_x_bytes_saved_per_step": shared_x_bytes(mats, x_groups, batch) * reps,
        "model_layers_per_step": reps, "stack_bytes": int(alg), "ms_per_step": ms_step,
        "us_per_matrix": 1e3 * ms_step / n_layers, "us_per_model_layer": 1e3 * ms_step / reps,
        "step_gbs": alg / (ms_step * 1e-3) / 1e9,
        "kernels": {k: {"ms": per_ms[k], "algorithmic_bytes": kb[k],
                        "gbs": kb[k] / (per_ms[k] * 1e-3) / 1e9 if per_ms[k] > 0 else None} for k in KERNELS},
        "world": world,
    }
    return res, (stack, x_all, y_all)


PREFILL_MATS = [(4096, 4096, 290, True)] * 4 + [(4096, 11008, 431, True)] * 2 + [(11008, 4096, 431, True)]
PREFILL_X_GROUPS = [0, 0, 0, 1, 2, 2, 3]   # q, k, v read one input; gate and up another


def measure_prefill(n_layers, M, steps, warmup, device, dist, seed=4321):
    """Llama-2-7B full linear stack at 0.3 BPW residual (4096^2 at s=290;
    4096<->11008 at s=431), M bf16 tokens per matrix, one forward_many per step.
    Within a model layer, q/k/v and gate/up read one input each, as in the
    model (PREFILL_X_GROUPS)."""
    import torch
    from latent_binary_factorization_b200 import layers as lbl, littlebit as lb
    gen = torch.Generator(device=device).manual_seed(seed)
    Ls, X, Y = [], [], []
    for _ in range(n_layers):
        xg = {}
        for (a, b, s, r), g in zip(PREFILL_MATS, PREFILL_X_GROUPS):
            Ls.append(lbl.random_layer(a, b, s, r, gen, device=device)[0])
            if g not in xg:
                xg[g] = torch.randn(M, a, generator=gen, device=device).to(torch.bfloat16)
            X.append(xg[g])
            Y.append(torch.empty(M, b, dtype=torch.bfloat16, device=device))
    stack = lb.Stack(Ls, X, Y)
    for _ in range(warmup):
        stack()
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        stack()
    t1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks([t0.elapsed_time(t1) / steps], device)[0]
    flops = sum(2 * M * s * (a + b) * (2 if r else 1) for a, b, s, r in PREFILL_MATS) * n_layers
    del stack, Ls, X, Y
    torch.cuda.empty_cache()
    return ms, flops


def run_ours(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = world > 1
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if dist:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    import latent_binary_factorization_b200.littlebit  # noqa: F401  fails loudly without the library
    props = torch.cuda.get_device_properties(device)
    l2 = props.L2_cache_size
    peak, peak_kind = load_peaks()

    sampler = ClockSampler(local)
    sampler.start()
    main, (stack, x_all, y_all) = measure_workload(args.workload, args.batch, args.steps, args.warmup, device,
                                                   dist, world, l2, l2_factor=args.l2_factor)
    # secondary figures: flat scalars (one level), so that a record keeping
    # only the line's scalar fields still holds them
    secondary = {}
    extras = {}
    if not args.no_extras:
        for name, b in (("70b_mlp_0.1bpw_residual", 1), ("70b_mlp_0.1bpw_single", 1),
                        ("7b_layer_0.1bpw_residual", 1), ("7b_attn_0.1bpw_residual", 1),
                        ("7b_attn_0.1bpw_single", 1), ("7b_attn_0.1bpw_residual", 4),
                        ("7b_attn_0.1bpw_residual", 16)):
            if name == args.workload and b == args.batch:
                continue
            r, held = measure_workload(name, b, max(10, args.steps // 2), args.warmup, device, dist, world, l2)
            del held
            torch.cuda.empty_cache()
            r["roofline_frac_step"] = r["step_gbs"] / peak
            extras[f"{name}_b{b}"] = r
            key = f"{name}_b{b}"
            secondary[f"{key}_us_per_model_layer"] = round(r["us_per_model_layer"], 4)
            secondary[f"{key}_step_hbm_frac"] = round(r["step_gbs"] / peak, 4)
            dk = max(KERNELS, key=lambda k: r["kernels"][k]["ms"])
            secondary[f"{key}_dominant_kernel_hbm_frac"] = round(r["kernels"][dk]["gbs"] / peak, 4)
        for b in (40, 130):
            extras[f"7b_attn_0.1bpw_residual_b{b}_mixed"] = measure_mixed(
                "7b_attn_0.1bpw_residual", b, max(5, args.steps // 4), args.warmup, device, dist, l2)
        extras["latency_single_layer"] = measure_latency(device)
        secondary["latency_single_layer_graph_us"] = extras["latency_single_layer"]["graph_us"]
    prefill = None
    if not args.no_prefill:
        psteps = max(20, args.steps // 10)
        pms, pflops = measure_prefill(args.prefill_layers, 2048, psteps, 3, device, dist)
        pk = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
            os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
        burst, sustained = float(pk.get("bf16_tflops", 1590.0)), float(pk.get("bf16_tflops_sustained", 1400.0))
        tf = pflops / (pms * 1e-3) / 1e12 * world
        prefill = {"workload": f"Llama-2-7B linear stack 0.3 BPW residual, {args.prefill_layers} layers, M=2048 bf16; "
                               "q/k/v and gate/up share their input",
                   "steps": psteps, "ms_per_step": round(pms, 4), "tflops": round(tf, 1), "unit": "TFLOP/s",
                   "algorithmic_flops_per_step": pflops, "bound": "tensor",
                   "peak_tflops": burst, "frac": round(tf / world / burst, 4),
                   "frac_of_sustained": round(tf / world / sustained, 4),
                   "peak_source": "measured (MEASURED_PEAKS.json bf16_tflops, burst)" if pk else "fallback",
                   "note": "step-level: operand preparation + both tcgen05 GEMMs, fp16 operands, fp32 accumulate"}
    clocks = sampler.stop()
    # the end-to-end pass runs after the clock sampler has stopped: it is bound
    # by host-side driver calls and PCIe copies, which nvidia-smi's polling
    # slows down, and it carries no clock-sensitive kernel time of its own
    e2e_steps = max(3, args.steps // 4)
    e2e_ms, h2d, d2h = time_e2e(stack, x_all, y_all, e2e_steps, 3, args.e2e_chunks)
    e2e_ms = max_over_ranks([e2e_ms], device)[0]
    del stack, x_all, y_all

    n_layers = main["layers_per_step"]
    model_layers = main["model_layers_per_step"]
    dom = max(KERNELS, key=lambda k: main["kernels"][k]["ms"])
    dom_bytes = main["kernels"][dom]["algorithmic_bytes"]
    dom_ms = main["kernels"][dom]["ms"]
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    traffic = traffic_record(dom, args.workload, model_layers)
    value = job_us_per_layer(main["ms_per_step"], model_layers, world)   # us per model layer over all ranks
    wl = WORKLOADS[args.workload]
    line = {
        "metric": METRIC,
        "value": round(value, 5),
        "unit": "us/layer",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(main["ms_per_step"], 5),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "i8",
        "dtype_note": "int8 tensor-core products (u8 sign planes x s8 hi/lo bytes of the 16-bit quantised vector), "
                      "int32 accumulation, fp32 scaling; fp16 x and y",
        "data": "synthetic: fair random signs, scales ~U[0.5,1.5]/sqrt(s), x ~ N(0,1) fp16",
        "config": {"workload": f"{wl['desc']}, decode batch {args.batch}, {model_layers} model layers "
                               f"({n_layers} matrices, {main['stack_bytes'] / 1e6:.0f} MB packed, inputs > L2, no flush)",
                   "layer": f"{len(wl['mats'])} matrices per model layer",
                   "batch": args.batch, "model_layers_per_gpu": model_layers, "matrices_per_gpu": n_layers,
                   "us_per_matrix": round(main["us_per_matrix"], 5), "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback", "algorithmic_bytes_per_launch": int(dom_bytes)},
        "step_roofline": {"achieved": round(main["step_gbs"], 1), "frac": round(main["step_gbs"] / peak, 4),
                          "kernels": {k: {"ms_per_step": round(main["kernels"][k]["ms"], 5),
                                          "gbs": round(main["kernels"][k]["gbs"], 1)
                                          if main["kernels"][k]["gbs"] else None} for k in KERNELS}},
        "step_hbm_frac": round(main["step_gbs"] / peak, 4),
        "e2e": {"value": round(job_us_per_layer(e2e_ms / e2e_steps, model_layers, world), 5), "unit": "us/layer",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "api": "littlebit_linear_forward_many_host (pinned host buffers)", "chunks": args.e2e_chunks,
                "note": "timed after the nvidia-smi clock sampler stopped"},
        "gpu_launches": 4 * args.steps,   # quantise, latent, finalize, output per step
        "clocks": clocks,
        "secondary": secondary,
        "prefill": prefill,
        "extras": extras,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, args.batch, budget_s=args.cpu_seconds)
    if dist:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# CPU oracle arm
# ---------------------------------------------------------------------------

def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _oracle_model_layers(workload, batch, seed, n_distinct):
    """n_distinct model layers of the workload (each a list of (paths, x) per
    matrix), drawn with the shared input generator for the CPU oracle."""
    from latent_binary_factorization_b200 import synth
    mats = WORKLOADS[workload]["mats"]
    out = []
    for i in range(n_distinct):
        out.append([(synth.layer(a, b, s, r, seed=seed, index=len(mats) * i + k),
                     synth.activations(batch, a, seed=seed, index=len(mats) * i + k))
                    for k, (a, b, s, r) in enumerate(mats)])
    return out


def cpu_baseline(workload, batch, budget_s=10.0, n_distinct=2):
    """Time the fp64 oracle (as it stands) on distinct model layers of the
    workload until about `budget_s` seconds of CPU work; returns us per model
    layer."""
    from oracle import littlebit_oracle as orc
    samples = _oracle_model_layers(workload, batch, 77, n_distinct)
    for paths, x in samples[0]:
        orc.factored_forward(x, paths)   # warm

    def timed(seconds):
        t0 = time.perf_counter()
        n = 0
        while True:
            for paths, x in samples[n % n_distinct]:
                orc.factored_forward(x, paths)
            n += 1
            if time.perf_counter() - t0 >= seconds and n >= 2:
                break
        return n, time.perf_counter() - t0

    n, dt = timed(budget_s)
    out = {"value": round(1e6 * dt / n, 3), "unit": "us/layer", "cores": _blas_threads(), "kind": "oracle",
           "sample": f"{n} forwards of {n_distinct} distinct model layers ({WORKLOADS[workload]['desc']}), "
                     f"batch {batch}, fp64 numpy, {dt:.1f} s", "nproc": os.cpu_count(), "cpu_model": _cpu_model()}
    try:   # the same oracle with its BLAS held to one thread
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1, user_api="blas"):
            n1, dt1 = timed(budget_s / 4)
        out["single_thread"] = {"value": round(1e6 * dt1 / n1, 3), "unit": "us/layer", "cores": 1,
                                "sample": f"{n1} model-layer forwards, {dt1:.1f} s"}
    except ImportError:
        pass
    return out


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import littlebit_oracle as orc
    n_distinct = 2
    samples = _oracle_model_layers(args.workload, args.batch, 88, n_distinct)

    def step(k):
        for paths, x in samples[k % n_distinct]:
            orc.factored_forward(x, paths)

    for k in range(args.warmup):
        step(k)
    t0 = time.perf_counter()
    for k in range(args.steps):
        step(k)
    dt = time.perf_counter() - t0
    value = 1e6 * dt / args.steps
    wl = WORKLOADS[args.workload]
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "us/layer", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * dt / args.steps, 3), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{wl['desc']}, decode batch {args.batch}; each step = one model layer "
                               f"({len(wl['mats'])} matrices) on the CPU oracle", "batch": args.batch},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 3), "unit": "us/layer", "kind": "oracle", "cores": _blas_threads(),
                         "sample": f"one model layer per step x {args.steps} steps, {n_distinct} distinct layers"},
        "e2e": {"value": round(value, 3), "unit": "us/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--no-extras", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill (tensor-core) measurement")
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="groups of layers whose host copies overlap the kernels in the end-to-end pass")
    ap.add_argument("--prefill-layers", type=int, default=32)
    ap.add_argument("--l2-factor", type=float, default=4.0,
                    help="stack size as a multiple of the L2 cache (>= 1 keeps inputs larger than L2)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
