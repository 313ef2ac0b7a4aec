#!/usr/bin/env python
"""Benchmark of the equivariant linear layers on B200.

Default workload: cyclic C_8 EQ-Linear at ViT-H width, bf16 I/O with fp32
accumulation, T = 131072 tokens (512 images x 256 tokens), 160 -> 160 fields of
8 group slots (1280 -> 1280 dense dims).  A step is one forward pass of the
whole layer (forward DFT, per-bin products, inverse DFT) over the step's
tokens; inputs already sit in HBM.  x + y are 671 MB per step, larger than
the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs its own T tokens (weak
scaling; the layer is token-parallel and needs no collective); the time is the
max over ranks and `value` counts the tokens of all ranks.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "EQ-Linear tokens/s and % of roofline (HBM or TC) at C_8, C=1280, bf16"
DEFAULT_WORKLOAD = "c8_t131072_160x160_bf16"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_SOURCES_DIR = "group_wise_dft_b200/csrc"   # every kernel and host-launch source


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--path", choices=("auto", "simt", "tc"), default="auto")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--graph", choices=("auto", "on", "off"), default="auto",
                    help="replay the K timed steps as one CUDA graph (auto: for workloads smaller "
                         "than L2, whose launches would otherwise wait on the host)")
    ap.add_argument("--pass", dest="which", choices=("forward", "backward_data", "weight_grad", "mlp"),
                    default="forward",
                    help="cyclic layers: time the backward data pass or the weight gradient instead "
                         "of the forward (same tokens); D8 layers: mlp times the Fourier-resident MLP "
                         "block (C -> 4C with the GELU round trip, then 4C -> C) on the workload's T, C")
    return ap.parse_args()


# ---------------------------------------------------------------- workloads


def workload(name):
    import workloads as synth
    if name in synth.CYCLIC_WORKLOADS:
        return synth.CYCLIC_WORKLOADS[name]
    if name in synth.D8_WORKLOADS:
        return synth.D8_WORKLOADS[name]
    raise SystemExit(f"unknown workload {name}")


def is_d8(w):
    return hasattr(w, "C")


def bytes_per_token(w, which="forward"):
    elt = 4 if w.dtype == "f32" else 2
    if is_d8(w):
        if which == "mlp":   # z in, hidden out and back in (4C), y out
            return 10 * w.C * elt
        return 2 * w.C * elt
    return (w.Cin + w.Cout) * w.N * elt


def flops_per_token(w, which="forward"):
    """Algorithmic FLOPs of the Fourier form: 2 * (real products per token)."""
    if is_d8(w):
        if which == "mlp":   # C -> 4C and 4C -> C, 3 C_in C_out / 16 products each
            return 2 * 2 * 3 * w.C * 4 * w.C // 16
        return 2 * 3 * w.C * w.C // 16
    real_bins = 2 if w.N % 2 == 0 and w.N > 1 else 1
    complex_bins = w.N // 2 + 1 - real_bins
    return 2 * (real_bins + 4 * complex_bins) * w.Cin * w.Cout


L2_BYTES = 126e6


def rotation_sets(step_bytes):
    """Buffer sets the timed steps rotate over: one when a step's x + y already
    exceed twice the L2, else enough for three L2s (at most 64), so that each
    step reads inputs that are not left in L2 by the step before."""
    if step_bytes >= 2 * L2_BYTES:
        return 1
    return int(min(64, math.ceil(3 * L2_BYTES / max(step_bytes, 1))))


def l2_note(w, R):
    mb = bytes_per_token(w) * w.T / 1e6
    if R == 1:
        return f"inputs larger than L2 ({mb:.0f} MB of x+y per step per GPU)"
    note = f"x+y are {mb:.3g} MB per step, less than L2: steps rotate over {R} buffer sets ({R * mb:.3g} MB)"
    if R * mb * 1e6 < 2 * L2_BYTES:
        note += "; the sets still fit in L2 (a latency-bound workload)"
    return note


def config_of(w, n_gpus, path_name, R=1):
    c = {"workload": w.name, "T_per_gpu": w.T, "dtype_io": w.dtype, "seed": w.seed,
         "parallelism": f"token-sharded x{n_gpus} (no collective)",
         "l2": l2_note(w, R),
         "kernel_path": path_name}
    if is_d8(w):
        c.update({"layer": "D8 Fourier-domain linear", "C": w.C, "fuse_gelu": w.fuse_gelu})
    else:
        c.update({"layer": f"cyclic C_{w.N} EQ-Linear", "fields_in": w.Cin, "fields_out": w.Cout,
                  "N": w.N, "dense_dims": f"{w.Cin * w.N}->{w.Cout * w.N}"})
    return c


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


WGRAD_SOURCES = ("wgrad_tc.cu", "simt_wgrad.cu", "wgrad_noalloc.cu")


def kernel_source_hash(weight_grad=False):
    """Hash of the sources under csrc (kernels and their host launches) that a
    pass runs: every file for the weight gradient, every file but the weight
    gradient's own for the other passes.  A recorded ncu traffic figure holds
    only while its hash is unchanged."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, KERNEL_SOURCES_DIR)
    for name in sorted(os.listdir(d)):
        if name.endswith((".cu", ".cuh", ".h")) and (weight_grad or name not in WGRAD_SOURCES):
            h.update(name.encode())
            h.update(open(os.path.join(d, name), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key):
    """Per-launch DRAM bytes from a committed ncu summary, only while the
    kernel sources still hash to what was profiled."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(kernel_key)
        if e and e.get("source_hash") == kernel_source_hash(kernel_key.endswith(":weight_grad")):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.dev = device_index
        self.path = None

    def start(self):
        import tempfile
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"unavailable": "nvidia-smi not runnable"}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    power = float(parts[2]) if parts[2] not in ("", "[N/A]") else float("nan")
                    rows.append((float(parts[0]), float(parts[1]), parts[3:], power))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"unavailable": "no samples"}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = set()
        for _, _, r, _ in rows:
            for n, v in zip(names, r[1:5]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        powers = [r[3] for r in rows if r[3] == r[3]]
        out = {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
               "sm_min_mhz": min(r[0] for r in rows), "reasons": sorted(reasons), "samples": len(rows)}
        if powers:
            out["power_w_max"] = max(powers)
        return out


# ---------------------------------------------------------------- oracle timing


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_rows_fn(w, which="forward"):
    """Closure running the oracle of the timed pass on a given number of rows of
    the workload (cycling through its first 8192 seeded rows)."""
    import numpy as np
    import torch
    import oracle
    import workloads as synth

    def f64(t):
        return t.float().numpy().astype(np.float64)

    n0 = min(w.T, 8192)
    if is_d8(w) and which == "mlp":
        z, w1, w2 = synth.d8_mlp_inputs(n0, w.C // 8, w.C // 2, w.torch_dtype, w.seed)
        rows, w1, w2 = f64(z), [f64(v) for v in w1], [f64(v) for v in w2]

        def one(m):
            oracle.d8_mlp_block(rows[:m], w1, w2)
    elif is_d8(w):
        x, *ws = synth.d8_inputs(n0, w.C, w.torch_dtype, w.seed)
        rows, ws64 = f64(x), [f64(v) for v in ws]

        def one(m):
            oracle.d8_forward(rows[:m], *ws64, fuse_gelu=w.fuse_gelu)
    elif which == "backward_data":
        _, W, dy = synth.cyclic_backward_inputs(n0, w.Cin, w.Cout, w.N, w.torch_dtype, w.seed)
        rows, W64 = f64(dy), f64(W)

        def one(m):
            oracle.cyclic_backward_data(rows[:m], W64)
    elif which == "weight_grad":
        x, _, dy = synth.cyclic_backward_inputs(n0, w.Cin, w.Cout, w.N, w.torch_dtype, w.seed)
        rows, dy64 = f64(x), f64(dy)

        def one(m):
            oracle.cyclic_weight_grad(rows[:m], dy64[:m])
    else:
        x, W = synth.cyclic_inputs(n0, w.Cin, w.Cout, w.N, w.torch_dtype, w.seed)
        rows, W64 = f64(x), f64(W)

        def one(m):
            oracle.cyclic_forward(rows[:m], W64)

    def run(n):
        reps = (n + len(rows) - 1) // len(rows)
        for r in range(reps):
            one(min(len(rows), n - r * len(rows)))
    return run


def time_oracle(w, budget_s=10.0, which="forward"):
    """Oracle throughput on a bounded sample: blocks of 1024 seeded token rows
    of the workload (cycling through its first 8192 rows) until ~budget_s of
    CPU work has run."""
    run = oracle_rows_fn(w, which)
    run(256)                                        # warm
    n, t0 = 0, time.perf_counter()
    chunk = 1024
    while True:
        run(chunk)
        n += chunk
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} token rows of {w.name} in blocks of 1024 (fp64 oracle of the {which} pass, "
                      f"numpy/BLAS), {dt:.1f} s"}


# ---------------------------------------------------------------- ranks


def rank_seed(w, rank):
    """Each rank draws its own token shard of the workload's shape (weak scaling)."""
    return w.seed + rank


def max_over_ranks(values, device):
    """Element-wise max over all ranks of a list of floats (identity on one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_tokens_per_s(tokens_per_rank, world, steps, elapsed_ms):
    """Whole-job throughput: the tokens of every rank over the slowest rank's time."""
    return tokens_per_rank * world * steps / (elapsed_ms / 1e3)


def reduce_weight_grad(dW):
    """Data-parallel training: each rank's dW covers its own tokens, the step's
    gradient is their sum over all ranks (one all-reduce of the Cout x Cin x N
    weight gradient; the one exchange step on this path)."""
    import torch.distributed as dist
    dist.all_reduce(dW, op=dist.ReduceOp.SUM)
    return dW


# ---------------------------------------------------------------- arms


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workload(args.workload)
    run = oracle_rows_fn(w, args.which)
    run(256)
    t0 = time.perf_counter()
    run(1024)
    per_row = (time.perf_counter() - t0) / 1024
    total_budget = 120.0
    rows = max(16, min(w.T, int(total_budget / max(1, args.steps + args.warmup) / per_row)))
    for _ in range(args.warmup):
        run(rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run(rows)
    dt = time.perf_counter() - t0
    value = rows * args.steps / dt
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(config_of(w, 1, "fp64 oracle on host cores"),
                           **({} if args.which == "forward" else {"pass": args.which})),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{rows} token rows of {w.name} per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    import group_wise_dft_b200 as eq
    import workloads as synth

    w = workload(args.workload)
    if is_d8(w) and args.which not in ("forward", "mlp"):
        raise SystemExit("--pass backward_data / weight_grad apply to the cyclic layers only")
    if not is_d8(w) and args.which == "mlp":
        raise SystemExit("--pass mlp applies to the D8 layers only")
    path = {"auto": eq.PATH_AUTO, "simt": eq.PATH_SIMT, "tc": eq.PATH_TC}[args.path]
    launches_per_step = 1
    if is_d8(w) and args.which == "mlp":
        F, Fh = w.C // 8, w.C // 2
        x_h, w1, w2 = synth.d8_mlp_inputs(w.T, F, Fh, w.torch_dtype, rank_seed(w, rank))
        x = x_h.to(dev)
        p1 = eq.d8_fourier_pack_weights(*[v.to(dev) for v in w1])
        p2 = eq.d8_fourier_pack_weights(*[v.to(dev) for v in w2])
        hid = torch.empty((w.T, Fh, 8), dtype=w.torch_dtype, device=dev)
        y = torch.empty_like(x)
        chosen = eq.PATH_SIMT
        mws_bytes = eq.d8_fourier_mlp_workspace_bytes(w.T, F, Fh, w.torch_dtype)
        mws = torch.empty(mws_bytes, dtype=torch.uint8, device=dev) if mws_bytes else None
        # expansion; contraction in column slices of 160 input fields plus their sum
        # when it has a workspace, else one CUDA-core launch
        launches_per_step = 1 + ((Fh + 159) // 160 + 1 if mws_bytes else 1)

        def step(xx=x, yy=y):
            eq.d8_fourier_mlp(xx, p1, p2, Fh, hidden=hid, y=yy, workspace=mws)
        pipe = eq.HostPipeline(lambda xx, yy: eq.d8_fourier_mlp(xx, p1, p2, Fh, y=yy),
                               (F, 8), (F, 8), w.torch_dtype, dev)
        wbytes = p1.numel() + p2.numel()
    elif is_d8(w):
        x_h, *ws = synth.d8_inputs(w.T, w.C, w.torch_dtype, rank_seed(w, rank))
        x = x_h.to(dev)
        Wp = eq.d8_pack_weights(*[v.to(dev) for v in ws])
        y = torch.empty_like(x)
        chosen = eq.d8_auto_path(w.C, w.torch_dtype) if path == eq.PATH_AUTO else path

        def step(xx=x, yy=y):
            eq.d8_forward(xx, Wp, fuse_gelu=w.fuse_gelu, y=yy, path=path)
        pipe = eq.HostPipeline(lambda xx, yy: eq.d8_forward(xx, Wp, fuse_gelu=w.fuse_gelu, y=yy, path=path),
                               (w.C // 8, 8), (w.C // 8, 8), w.torch_dtype, dev)
        wbytes = Wp.numel()
    elif args.which == "forward":
        x_h, W_h = synth.cyclic_inputs(w.T, w.Cin, w.Cout, w.N, w.torch_dtype, rank_seed(w, rank))
        x = x_h.to(dev)
        Ws = eq.cyclic_weight_spectrum(W_h.to(dev))
        y = torch.empty((w.T, w.Cout, w.N), dtype=w.torch_dtype, device=dev)
        chosen = eq.cyclic_auto_path(w.N, w.Cin, w.Cout, w.torch_dtype) if path == eq.PATH_AUTO else path

        # C_16 layers take the two-pass tensor-core path when given a workspace
        need = eq.cyclic_forward_workspace_bytes(w.T, w.N, w.Cin, w.Cout, w.torch_dtype)
        fws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev) if need else None
        if need and path != eq.PATH_SIMT:
            chosen = eq.PATH_TC

        if fws is not None and chosen == eq.PATH_TC:
            launches_per_step = 3   # fold, the cyclic pass, the negacyclic pass with the combine

        def fwd(xx, yy):
            if fws is not None:
                eq.cyclic_forward_ws(xx, Ws, w.Cout, y=yy, path=path, workspace=fws)
            else:
                eq.cyclic_forward(xx, Ws, w.Cout, y=yy, path=path)

        def step(xx=x, yy=y):
            fwd(xx, yy)
        pipe = eq.HostPipeline(fwd, (w.Cin, w.N), (w.Cout, w.N), w.torch_dtype, dev)
        wbytes = w.Cin * w.Cout * w.N * (4 if w.dtype == "f32" else 2)
    elif args.which == "backward_data":
        # dy [T, Cout, N] -> dx [T, Cin, N]: the layer Cout -> Cin with the adjoint spectrum
        _, W_h, dy_h = synth.cyclic_backward_inputs(w.T, w.Cin, w.Cout, w.N, w.torch_dtype, rank_seed(w, rank))
        x_h = dy_h
        x = dy_h.to(dev)
        Wa = eq.cyclic_weight_spectrum_adjoint(W_h.to(dev))
        y = torch.empty((w.T, w.Cin, w.N), dtype=w.torch_dtype, device=dev)
        chosen = eq.cyclic_auto_path(w.N, w.Cout, w.Cin, w.torch_dtype) if path == eq.PATH_AUTO else path

        def step(xx=x, yy=y):
            eq.cyclic_backward_data(xx, Wa, w.Cin, dx=yy, path=path)
        pipe = eq.HostPipeline(lambda xx, yy: eq.cyclic_backward_data(xx, Wa, w.Cin, dx=yy, path=path),
                               (w.Cout, w.N), (w.Cin, w.N), w.torch_dtype, dev)
        wbytes = w.Cin * w.Cout * w.N * (4 if w.dtype == "f32" else 2)
    else:
        # x [T, Cin, N] and dy [T, Cout, N] -> dW [Cout, Cin, N]
        xw_h, _, dy_h = synth.cyclic_backward_inputs(w.T, w.Cin, w.Cout, w.N, w.torch_dtype, rank_seed(w, rank))
        x_h = xw_h
        x = xw_h.to(dev)
        dyd = dy_h.to(dev)
        y = torch.empty((w.Cout, w.Cin, w.N), dtype=w.torch_dtype, device=dev)
        wsp = torch.empty(max(eq.cyclic_weight_grad_workspace_bytes(w.T, w.N, w.Cin, w.Cout, w.torch_dtype), 16),
                          dtype=torch.uint8, device=dev)
        tc_ok = w.N == 8 and w.dtype == "bf16" and min(w.Cin, w.Cout) >= 8
        chosen = eq.PATH_TC if tc_ok and path != eq.PATH_SIMT else eq.PATH_SIMT
        launches_per_step = 2   # per-split partials, then the reduction and inverse

        def step(xx=x, yy=y):
            eq.cyclic_weight_grad(xx[0], xx[1], dW=yy, workspace=wsp, path=path)
            if world > 1:
                reduce_weight_grad(yy)
        x = (x, dyd)
        pipe = None
        wbytes = w.Cin * w.Cout * w.N * (4 if w.dtype == "f32" else 2)
    path_name = {eq.PATH_SIMT: "simt", eq.PATH_TC: "tcgen05"}[chosen]
    if is_d8(w) and args.which == "mlp":
        tc_expand = w.dtype == "bf16" and (w.C // 8) % 16 == 0 and w.C // 8 <= 160
        path_name = ("tcgen05 (contraction in column slices)" if tc_expand and mws_bytes
                     else "tcgen05 expand + simt contract" if tc_expand else "simt")
    # inputs smaller than L2 rotate over several buffer sets (see rotation_sets)
    R = rotation_sets(bytes_per_token(w, args.which) * w.T)
    xs = [x] + [tuple(v.clone() for v in x) if isinstance(x, tuple) else x.clone() for _ in range(R - 1)]
    ys = [y] + [torch.empty_like(y) for _ in range(R - 1)]
    torch.cuda.synchronize()

    for i in range(args.warmup):
        step(xs[i % R], ys[i % R])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    stream = torch.cuda.current_stream(dev)
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(getattr(torch.cuda.get_device_properties(dev), "uuid", local))
    if hasattr(torch.cuda.get_device_properties(dev), "uuid"):
        sampler.dev = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    # small workloads: the K steps as one CUDA graph (the same library calls,
    # captured once), so the device is not left waiting on the host between launches
    use_graph = args.graph == "on" or (args.graph == "auto" and R > 1)
    use_graph = use_graph and args.which != "weight_grad"   # that pass may hold an NCCL call
    graph = None
    if use_graph:
        gs = torch.cuda.Stream(dev)
        gs.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gs):
            for k in range(K):
                step(xs[k % R], ys[k % R])
        torch.cuda.synchronize()
        graph.replay()   # one untimed replay
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    sampler.start()
    torch.cuda.synchronize()
    t_start.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for k in range(K):
            ev[k][0].record(stream)
            step(xs[k % R], ys[k % R])
            ev[k][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = t_start.elapsed_time(t_end)
    per_launch = total_ms / K if graph is not None else statistics.mean(a.elapsed_time(b) for a, b in ev)
    elapsed_ms, launch_ms = max_over_ranks([total_ms, per_launch], dev)
    del graph
    ms_per_step = elapsed_ms / K
    value = job_tokens_per_s(w.T, world, K, elapsed_ms)

    # end to end through the public API with host buffers: every step copies x
    # in from pinned host memory and y back out (HostPipeline overlaps the two
    # PCIe directions and the kernel, chunk by chunk)
    E = max(3, args.e2e_steps)
    if pipe is not None:
        x_pin = x_h.pin_memory()
        y_pin = torch.empty(tuple(y.shape), dtype=y.dtype).pin_memory()
        for _ in range(3):
            pipe.run(x_pin, y_pin)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(E):
            pipe.run(x_pin, y_pin)
        e1.record(stream)
        torch.cuda.synchronize()
        (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1)], dev)
        if world > 1:
            dist.barrier()
        e2e_value = job_tokens_per_s(w.T, world, E, e2e_ms)
        e2e = {"value": e2e_value, "unit": "tokens/s",
               "h2d_bytes_per_step": x.numel() * x.element_size(),
               "d2h_bytes_per_step": y.numel() * y.element_size()}
    else:
        # the weight gradient reduces over every token, so there is no chunked
        # pipeline: each step copies all of x and dy in, runs, copies dW out
        xh_pin, dyh_pin = x_h.pin_memory(), dy_h.pin_memory()
        dW_pin = torch.empty(tuple(y.shape), dtype=y.dtype).pin_memory()
        xd, dyd2 = torch.empty_like(xs[0][0]), torch.empty_like(xs[0][1])

        def e2e_step():
            xd.copy_(xh_pin, non_blocking=True)
            dyd2.copy_(dyh_pin, non_blocking=True)
            eq.cyclic_weight_grad(xd, dyd2, dW=y, workspace=wsp, path=path)
            if world > 1:
                reduce_weight_grad(y)
            dW_pin.copy_(y, non_blocking=True)
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(E):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1)], dev)
        if world > 1:
            dist.barrier()
        e2e = {"value": job_tokens_per_s(w.T, world, E, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": xd.numel() * xd.element_size() + dyd2.numel() * dyd2.element_size(),
               "d2h_bytes_per_step": y.numel() * y.element_size(),
               "note": "whole x and dy copied in, then the kernels, then dW out (no overlap)"}

    hbm_peak, tc_peak, tc_sustained, peak_src = measured_peaks()
    alg_bytes = w.T * bytes_per_token(w, args.which) + wbytes
    achieved_gbs = alg_bytes / (launch_ms / 1e3) / 1e9
    alg_flops = w.T * flops_per_token(w, args.which)
    achieved_tflops = alg_flops / (launch_ms / 1e3) / 1e12
    t_hbm = alg_bytes / (hbm_peak * 1e9)
    t_tc = alg_flops / (tc_peak * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    kernel_key = f"{path_name}:{w.name}" + ("" if args.which == "forward" else f":{args.which}")
    traffic = recorded_traffic(kernel_key)
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved_gbs / hbm_peak, "traffic": traffic, "peak_source": peak_src,
                "algorithmic_bytes_per_launch": alg_bytes}
    else:
        roof = {"bound": "tensor", "achieved": achieved_tflops, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": achieved_tflops / tc_peak, "traffic": traffic, "peak_source": peak_src,
                "algorithmic_flops_per_launch": alg_flops}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": dict(config_of(w, world, path_name, R), **({} if args.which == "forward" else {"pass": args.which}),
                           **({"exchange": "NCCL all-reduce (sum) of dW per step"}
                              if args.which == "weight_grad" and world > 1 else {})),
            "roofline": roof,
            "roofline_fraction_of_max_bound": max(t_hbm, t_tc) / (launch_ms / 1e3),
            "tensor_pipe": {"achieved_tflops": achieved_tflops, "peak_tflops": tc_peak,
                            "frac": achieved_tflops / tc_peak, "algorithmic_flops_per_launch": alg_flops},
            "effective_dense_tflops": (2 * w.T * ((8 if args.which == "mlp" else 1) * w.C * w.C if is_d8(w)
                                                  else w.Cin * w.N * w.Cout * w.N))
            / (launch_ms / 1e3) / 1e12,
            "kernel_ms_per_launch": launch_ms,
            "timing": ("one CUDA graph of the K steps, replayed once; per-step time = total / K"
                       if use_graph else "eager launches, CUDA events around each step"),
            "clocks": clocks,
            "e2e": e2e,
            "gpu_launches": K * launches_per_step}
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = time_oracle(w, which=args.which)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def free_port():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launcher_command(argv, gpus, port, script=None):
    """torchrun command that starts one rank per GPU on this node (127.0.0.1
    rendezvous) running `script` (this file) with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr", "127.0.0.1", f"--master-port={port}",
            script or os.path.abspath(__file__), *argv]


def main():
    args = parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # started as a single process: start the N ranks here, one per GPU
        cmd = ["timeout", "-k", "60", "1800"] + launcher_command(sys.argv[1:], args.gpus, free_port())
        return subprocess.call(cmd)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
