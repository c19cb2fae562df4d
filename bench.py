"""Benchmark of the GradLev scan: forward + reverse scan tokens/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config IDX] [--no-e2e] [--no-cpu-baseline]
    python bench.py --decode [--steps K] [--warmup W] [--T TOKENS_PER_CALL]
    python bench.py --consistency [--steps K] [--warmup W] [--config IDX]
    python bench.py --mlp2 [--steps K] [--warmup W]

One step = one forward scan (with state checkpoints) + one reverse scan over
one batch of the workload, i.e. every step of the hot path. The default
workload is the bf16 forward+backward scan B=8, H=16, T=4096, d_in=d_out=128
with alpha = 1 - 10^U(-4,-1). Inputs are synthetic, drawn by the seeded
generator, and resident in HBM before the timed region (working set larger
than the 126 MB L2, so no flush is done between steps).

With N > 1 (launched by torch.distributed.run) every rank runs its own batch
(weak scaling); the only exchange is the dW0 all-reduce over ranks (dW0 sums
over the batch). Time is taken on the device with CUDA events, max over ranks.

``--impl reference`` times the float64 CPU oracle on a bounded sample of the
same workload on rank 0 (other ranks exit at once).

``--decode`` measures the deployment decode step instead and prints its own
line. The shape is B8 H16 d128 bf16, one token per call unless --T says more.
The states and weights of 16 layers are rotated, 134 MB in all, more than the
L2. The call loop is captured in a CUDA graph; the plain-launch time is
reported beside it.

``--consistency`` times gradlev_consistency_step on the workload's shape. One
call is a whole training step from predicted costates: the forward, the
reconstructed costates and losses, the reverse scan, and the consistency
gradient. It prints its own line.

``--mlp2`` times gradlev_mlp2_recon, the two-layer reconstruction of the
synthetic test, at bf16 B8 H16 T4096 with d_x = d_h = d_y = 128, and prints
its own line.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GradLev scan fwd+bwd tokens/s and % of roofline on 1 B200 (B8 H16 T4096 d128)"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--config", type=int, default=3)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=15.0,
                   help="target CPU work of the oracle sample")
    p.add_argument("--B", type=int, default=None, help="override B (reduced profiling case)")
    p.add_argument("--H", type=int, default=None, help="override H (reduced profiling case)")
    p.add_argument("--T", type=int, default=None, help="override T (reduced profiling case)")
    p.add_argument("--decode", action="store_true", help="time the deployment decode step")
    p.add_argument("--consistency", action="store_true",
                   help="time the consistency training step")
    p.add_argument("--mlp2", action="store_true", help="time the two-layer reconstruction")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def alg_bytes(cfg, es, passes=("fwd", "bwd")):
    """Algorithmic bytes: every input read once, every output written once."""
    N = cfg.B * cfg.H * cfg.T
    di, do = cfg.d_in, cfg.d_out
    w = cfg.H * di * do * 4
    out = {}
    out["fwd"] = N * (di + 2 * do) * es + N * 8 + w
    out["bwd"] = N * (2 * di + 3 * do) * es + N * 16 + 2 * w
    return out


def alg_flops(cfg):
    N = cfg.B * cfg.H * cfg.T
    return {"fwd": 4 * N * cfg.d_in * cfg.d_out, "bwd": 12 * N * cfg.d_in * cfg.d_out}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": ["no samples"]}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def kernel_traffic(cfg, dom):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary, or
    None when the kernel source changed since the counters were taken, or when the
    record is for another call or workload."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None, None
    with open(path) as f:
        d = json.load(f)
    src = os.path.join(ROOT, d.get("source", ""))
    if not os.path.exists(src):
        return None, None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if h != d.get("source_sha256"):
        return None, d.get("kernel")
    w = d.get("workload", {})
    shape = {"B": cfg.B, "H": cfg.H, "T": cfg.T, "d_in": cfg.d_in, "d_out": cfg.d_out}
    if d.get("call") != dom or w != shape:
        return None, d.get("kernel")
    return d.get("bytes_per_launch"), d.get("kernel")


def _oracle_sample(cfg, seconds):
    """Draw a bounded sample of the workload's scans sized for ~`seconds` of wall time
    of the oracle on this host's cores."""
    import oracle
    from token_weight_scans_b200 import inputs
    nth = oracle.max_threads()
    Tp = min(cfg.T, 128)
    d = inputs.draw(1, 1, Tp, cfg.d_in, cfg.d_out, dtype=cfg.dtype, alpha_mode=cfg.alpha_mode,
                    seed=1)
    d = {k: v.astype(np.float64) for k, v in d.items()}
    t0 = time.perf_counter()
    oracle.fwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"], nthreads=1)
    oracle.bwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"], d["dy"], nthreads=1)
    per_tok = (time.perf_counter() - t0) / Tp
    budget = seconds * nth / max(per_tok, 1e-9)          # head-tokens
    n_scans = int(min(cfg.B * cfg.H, max(1, budget // cfg.T)))
    T = cfg.T if budget >= cfg.T else max(64, int(budget))
    d = inputs.draw(n_scans, 1, T, cfg.d_in, cfg.d_out, dtype=cfg.dtype,
                    alpha_mode=cfg.alpha_mode, seed=2)
    return {k: v.astype(np.float64) for k, v in d.items()}, nth


def _time_oracle(cfg, d, nth):
    import oracle
    t0 = time.perf_counter()
    oracle.fwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"])
    oracle.bwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"], d["dy"])
    wall = time.perf_counter() - t0
    n_scans, T = d["x"].shape[0], d["x"].shape[2]
    head_tokens = n_scans * T
    # tokens/s in the metric's unit: a token is one position across all H heads
    return {"value": head_tokens / cfg.H / wall, "unit": "tokens/s", "cores": nth,
            "kind": "oracle",
            "sample": f"{n_scans} scans x T={T} (d_in={cfg.d_in}, d_out={cfg.d_out}) fwd+bwd, "
                      f"float64 oracle, OpenMP over scans on {nth} threads; {head_tokens} "
                      f"head-tokens in {wall:.2f} s; tokens/s = head-tokens / H / wall"}


def cpu_baseline(cfg, seconds):
    """Time the float64 oracle (fwd + bwd) on a bounded sample of the workload's scans."""
    d, nth = _oracle_sample(cfg, seconds)
    return _time_oracle(cfg, d, nth)


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = min(6.0, max(1.0, 150.0 / max(1, args.steps + args.warmup)))
    d, nth = _oracle_sample(cfg, per_step)
    vals, r = [], None
    for i in range(args.warmup + args.steps):
        r = _time_oracle(cfg, d, nth)
        if i >= args.warmup:
            vals.append(r["value"])
    value = float(np.median(vals))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": cfg.tokens / value * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "T": cfg.T,
                       "d_in": cfg.d_in, "d_out": cfg.d_out, "passes": "fwd+bwd",
                       "l2": "CPU run of a bounded sample; no GPU involved"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r["cores"],
                             "kind": "oracle", "sample": r["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_decode(args):
    """Deployment decode: one gradlev_decode_step call per layer per token."""
    import torch

    import token_weight_scans_b200 as tw
    from token_weight_scans_b200 import build as tw_build
    from token_weight_scans_b200 import inputs
    torch.cuda.set_device(0)
    tw_build.build()
    tw.lib()
    B, H, d = args.B or 8, args.H or 16, 128
    T = args.T or 1
    layers = 16
    dev = torch.device("cuda", 0)
    lay = []
    for l in range(layers):
        dr = inputs.draw(B, H, T, d, d, dtype="bf16", alpha_mode="sigmoid", seed=5000 + l,
                         with_v=True)
        t = {k: torch.from_numpy(v).to(dev) for k, v in dr.items()}
        for k in ("x", "v"):
            t[k] = t[k].to(torch.bfloat16)
        t["S"] = torch.zeros((B, H, d, d), dtype=torch.float32, device=dev)
        t["y"] = torch.empty((B, H, T, d), dtype=torch.bfloat16, device=dev)
        t["g"] = torch.empty_like(t["y"])
        lay.append(t)

    def call(t):
        tw.gradlev_decode_step(t["x"], t["v"], t["eta"], t["alpha"], t["W0"], t["S"], y=t["y"],
                               g=t["g"])

    K = max(1, args.steps) * layers
    for i in range(max(3, args.warmup) * layers):
        call(lay[i % layers])
    torch.cuda.synchronize()
    s0, e0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for i in range(K):
        call(lay[i % layers])
    e0.record()
    torch.cuda.synchronize()
    plain_us = s0.elapsed_time(e0) * 1e3 / K
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for i in range(K):
                call(lay[i % layers])
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    s1, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 5
    s1.record()
    for _ in range(reps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    us = s1.elapsed_time(e1) * 1e3 / (reps * K)
    peaks, peak_src = load_peaks()
    # algorithmic bytes of one call: S read and written, W0 read, the token vectors
    byt = B * H * d * d * 4 * 2 + H * d * d * 4 + B * H * T * d * 2 * 4 + B * H * T * 8
    gbs = byt / (us * 1e-6) / 1e9
    line = {"metric": "GradLev deployment decode: tokens/s through 16 adapted layers on 1 B200 "
                      f"(B{B} H{H} d{d} bf16, {T} token(s) per call)",
            "value": B * T / (us * 1e-6 * layers), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "us_per_call": us,
            "us_per_call_plain_launch": plain_us, "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic (seeded generator)",
            "config": {"workload": "decode", "B": B, "H": H, "T_per_call": T, "d_in": d,
                       "d_out": d, "layers": layers, "cuda_graph": True,
                       "l2": f"no flush: {layers} layers' S and W0 "
                             f"({layers * (B * H + H) * d * d * 4 / 1e6:.0f} MB) > 126 MB L2"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                         "alg_bytes_per_launch": byt, "kernel": "decode_kernel",
                         "peak_source": peak_src},
            "clocks": clk, "gpu_launches": reps * K}
    print(json.dumps(line), flush=True)


def run_consistency(args):
    """gradlev_consistency_step on the workload's shape (inputs resident in HBM)."""
    import torch

    import token_weight_scans_b200 as tw
    from token_weight_scans_b200 import build as tw_build
    from token_weight_scans_b200 import inputs
    torch.cuda.set_device(0)
    tw_build.build()
    tw.lib()
    cfg = inputs.CONFIGS[args.config]
    B, H, T, di, do = cfg.B, cfg.H, cfg.T, cfg.d_in, cfg.d_out
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    es = 2 if cfg.dtype == "bf16" else 4
    d = inputs.draw(B, H, T, di, do, dtype=cfg.dtype, alpha_mode=cfg.alpha_mode, seed=77,
                    with_v=True)
    t = {k: torch.from_numpy(v).cuda() for k, v in d.items()}
    for k in ("x", "g", "v"):
        t[k] = t[k].to(tdt)
    code = tw.BF16 if cfg.dtype == "bf16" else tw.F32
    ws = torch.empty(tw.gradlev_consistency_workspace_bytes(B, H, T, di, do, code),
                     dtype=torch.uint8, device="cuda")
    out = None

    def step():
        nonlocal out
        out = tw.gradlev_consistency_step(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], t["v"],
                                          1.0, workspace=ws, out=out)
        return tw.gradlev_last_launch_count()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    s0, e0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    s0.record()
    for _ in range(args.steps):
        launches += step()
    e0.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = s0.elapsed_time(e0) / args.steps
    peaks, peak_src = load_peaks()
    N = B * H * T
    ab = alg_bytes(cfg, es)
    # residual: y, ghat, v read, gtil and dv written, two losses; finish: dg, ghat, gtil
    # read, dg written
    extra = N * do * es * (5 + 4) + N * 8
    byt = ab["fwd"] + ab["bwd"] + extra
    gbs = byt / (ms * 1e-3) / 1e9
    line = {"metric": f"GradLev consistency training step tokens/s on 1 B200 ({cfg.name})",
            "value": B * T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "dtype": cfg.dtype, "data": "synthetic (seeded generator)",
            "config": {"workload": "consistency step, " + cfg.name, "B": B, "H": H, "T": T,
                       "d_in": di, "d_out": do,
                       "l2": f"no flush: {byt / 1e6:.0f} MB per step > 126 MB L2"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                         "alg_bytes_per_step": byt, "peak_source": peak_src},
            "clocks": clk, "gpu_launches": launches}
    print(json.dumps(line), flush=True)


def run_mlp2(args):
    """gradlev_mlp2_recon at bf16 B8 H16 T4096, d_x = d_h = d_y = 128."""
    import torch

    import token_weight_scans_b200 as tw
    from token_weight_scans_b200 import build as tw_build
    torch.cuda.set_device(0)
    tw_build.build()
    tw.lib()
    B, H, T = args.B or 8, args.H or 16, args.T or 4096
    d = 128
    g = torch.Generator(device="cuda").manual_seed(91)
    rn = lambda *s: torch.randn(*s, generator=g, device="cuda")
    bf = torch.bfloat16
    x, v = rn(B, H, T, d).to(bf), rn(B, H, T, d).to(bf)
    g1, g2 = (0.1 * rn(B, H, T, d)).to(bf), (0.1 * rn(B, H, T, d)).to(bf)
    eta = 0.5 / d * torch.rand(B, H, T, generator=g, device="cuda")
    alpha = 0.9 + 0.099 * torch.rand(B, H, T, generator=g, device="cuda")
    W1, W2 = rn(H, d, d) / d ** 0.5, rn(H, d, d) / d ** 0.5
    ws = torch.empty(tw.gradlev_mlp2_workspace_bytes(B, H, T, d, d, d, tw.BF16),
                     dtype=torch.uint8, device="cuda")
    out = None

    def step():
        nonlocal out
        out = tw.gradlev_mlp2_recon(x, g1, g2, v, eta, alpha, W1, W2, workspace=ws, out=out)
        return tw.gradlev_last_launch_count()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    s0, e0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    s0.record()
    for _ in range(args.steps):
        launches += step()
    e0.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = s0.elapsed_time(e0) / args.steps
    N = B * H * T
    # algorithmic bytes: two forward scans (x, g1hat, a; h, g2hat, y), tanh (a in, h out),
    # the reconstruction (x, h, g2hat, y, v in; g2til, g1til out) and dW1
    byt = N * d * 2 * (3 + 3 + 2 + 7) + 4 * N * 8 + 2 * H * d * d * 4 + B * H * d * d * 4
    flops = 2 * N * d * d * (2 + 2) + 2 * N * d * d * 4  # scans, then W2^T u, S2^T u, carry, dW1
    peaks, peak_src = load_peaks()
    line = {"metric": "GradLev two-layer reconstruction tokens/s on 1 B200 "
                      f"(B{B} H{H} T{T} d128 bf16)",
            "value": B * T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic (seeded generator)",
            "config": {"workload": "mlp2 reconstruction", "B": B, "H": H, "T": T, "d_x": d,
                       "d_h": d, "d_y": d},
            "roofline": {"bound": "hbm", "achieved": byt / (ms * 1e-3) / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": byt / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "alg_bytes_per_step": byt, "alg_flops_per_step": flops,
                         "peak_source": peak_src},
            "clocks": clk, "gpu_launches": launches}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.mlp2:
        return run_mlp2(args)
    if args.decode:
        return run_decode(args)
    if args.consistency:
        return run_consistency(args)
    from token_weight_scans_b200 import inputs
    cfg = inputs.CONFIGS[args.config]
    over = {k: getattr(args, k) for k in ("B", "H", "T") if getattr(args, k) is not None}
    if over:
        import dataclasses
        cfg = dataclasses.replace(cfg, name=cfg.name + " reduced to " + " ".join(
            f"{k}={v}" for k, v in over.items()), **over)
    if args.impl == "reference":
        return run_reference(args, cfg)

    import torch
    import torch.distributed as dist

    import token_weight_scans_b200 as tw
    from token_weight_scans_b200 import build as tw_build
    from token_weight_scans_b200 import multirank

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    if rank == 0:
        tw_build.build()
    if world > 1:
        dist.barrier()
    tw.lib()

    code = tw.BF16 if cfg.dtype == "bf16" else tw.F32
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    es = 2 if cfg.dtype == "bf16" else 4
    do_bwd = "bwd" in cfg.passes
    B, H, T, di, do = cfg.B, cfg.H, cfg.T, cfg.d_in, cfg.d_out
    if tw.gradlev_scan_supported(B, H, T, di, do, code) != 0:
        raise SystemExit(f"workload {cfg.name} is not supported by the library")

    # inputs: each rank its own seeded batch (weak scaling)
    d = inputs.draw(B, H, T, di, do, dtype=cfg.dtype, alpha_mode=cfg.alpha_mode,
                    seed=multirank.rank_seed(cfg.index, rank))
    host = {}
    for k, v in d.items():
        t = torch.from_numpy(v)
        if k in ("x", "g", "dy"):
            t = t.to(tdt)
        host[k] = t.pin_memory()
    dv = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
    del d
    y = torch.empty((B, H, T, do), dtype=tdt, device=dev)
    gr = dict(dx=torch.empty_like(dv["x"]), dg=torch.empty_like(dv["g"]),
              deta=torch.empty((B, H, T), device=dev), dalpha=torch.empty((B, H, T), device=dev),
              dW0=torch.empty((H, do, di), device=dev))
    ck = torch.empty(tw.gradlev_scan_ckpt_bytes(B, H, T, di, do, code), dtype=torch.uint8,
                     device=dev)
    ws = torch.empty(max(tw.gradlev_scan_workspace_bytes(B, H, T, di, do, code, 1),
                         tw.gradlev_scan_workspace_bytes(B, H, T, di, do, code, 0)),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    launches = [0]

    def step(xs=None):
        src = dv if xs is None else xs
        tw.gradlev_scan_fwd(src["x"], src["g"], src["eta"], src["alpha"], src["W0"], y=y,
                            ckpt=ck if do_bwd else None, workspace=ws)
        launches[0] += tw.gradlev_last_launch_count()
        if do_bwd:
            tw.gradlev_scan_bwd(src["x"], src["g"], src["eta"], src["alpha"], src["W0"],
                                src["dy"], ckpt=ck, workspace=ws, out=gr)
            launches[0] += tw.gradlev_last_launch_count()
            multirank.allreduce_dW0(gr["dW0"], dist)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # per-call events for the dominant-kernel roofline, inside the timed region
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    launches[0] = 0
    start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        tw.gradlev_scan_fwd(dv["x"], dv["g"], dv["eta"], dv["alpha"], dv["W0"], y=y,
                            ckpt=ck if do_bwd else None, workspace=ws)
        launches[0] += tw.gradlev_last_launch_count()
        ev[i][1].record(stream)
        if do_bwd:
            tw.gradlev_scan_bwd(dv["x"], dv["g"], dv["eta"], dv["alpha"], dv["W0"], dv["dy"],
                                ckpt=ck, workspace=ws, out=gr)
            launches[0] += tw.gradlev_last_launch_count()
        ev[i][2].record(stream)
        if do_bwd:
            multirank.allreduce_dW0(gr["dW0"], dist)
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = start.elapsed_time(end)
    fwd_ms = float(np.mean([a.elapsed_time(b) for a, b, _ in ev]))
    bwd_ms = float(np.mean([b.elapsed_time(c) for _, b, c in ev])) if do_bwd else 0.0
    ms = multirank.max_over_ranks(ms, dist, device=dev)
    gpu_launches = launches[0]

    # e2e through the public API with host buffers: every step copies its inputs in from
    # pinned host memory, runs the scan and copies its results out. Two device buffer sets
    # and three streams let the H2D copy of step i + 1 and the D2H copy of step i - 1 overlap
    # the scan of step i, as a deployment would; the checkpoints and the workspace are shared
    # (the scans run in order on one stream).
    e2e = None
    if not args.no_e2e:
        out_host = {"y": torch.empty_like(y, device="cpu").pin_memory()}
        if do_bwd:
            out_host.update({k: torch.empty_like(v, device="cpu").pin_memory()
                             for k, v in gr.items()})
        in_keys = ("x", "g", "eta", "alpha", "W0") + (("dy",) if do_bwd else ())
        h2d = sum(host[k].numel() * host[k].element_size() for k in in_keys)
        d2h = sum(v.numel() * v.element_size() for v in out_host.values())
        e_steps = max(3, min(args.steps, 10))
        sets = [(dv, y, gr),
                ({k: torch.empty_like(v) for k, v in dv.items()}, torch.empty_like(y),
                 {k: torch.empty_like(v) for k, v in gr.items()})]
        s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))

        def e2e_run(nsteps, ev_start=None, ev_end=None):
            done_cmp, done_out = [None, None], [None, None]
            if ev_start is not None:
                ev_start.record(s_in)
            for i in range(nsteps):
                k = i % 2
                dvs, ys, grs = sets[k]
                with torch.cuda.stream(s_in):  # this set's previous scan has read its inputs
                    if done_cmp[k] is not None:
                        s_in.wait_event(done_cmp[k])
                    for key in in_keys:
                        dvs[key].copy_(host[key], non_blocking=True)
                    e_in = torch.cuda.Event()
                    e_in.record(s_in)
                with torch.cuda.stream(s_cmp):  # and its previous results are out
                    s_cmp.wait_event(e_in)
                    if done_out[k] is not None:
                        s_cmp.wait_event(done_out[k])
                    tw.gradlev_scan_fwd(dvs["x"], dvs["g"], dvs["eta"], dvs["alpha"], dvs["W0"],
                                        y=ys, ckpt=ck if do_bwd else None, workspace=ws,
                                        stream=s_cmp)
                    if do_bwd:
                        tw.gradlev_scan_bwd(dvs["x"], dvs["g"], dvs["eta"], dvs["alpha"],
                                            dvs["W0"], dvs["dy"], ckpt=ck, workspace=ws, out=grs,
                                            stream=s_cmp)
                        multirank.allreduce_dW0(grs["dW0"], dist)
                    done_cmp[k] = torch.cuda.Event()
                    done_cmp[k].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(done_cmp[k])
                    out_host["y"].copy_(ys, non_blocking=True)
                    if do_bwd:
                        for key, v in grs.items():
                            out_host[key].copy_(v, non_blocking=True)
                    done_out[k] = torch.cuda.Event()
                    done_out[k].record(s_out)
            if ev_end is not None:
                s_out.wait_stream(s_cmp)
                s_out.wait_stream(s_in)
                ev_end.record(s_out)

        e2e_run(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_run(e_steps, s2, e2)
        torch.cuda.synchronize()
        ems = s2.elapsed_time(e2) / e_steps
        ems = multirank.max_over_ranks(ems, dist, device=dev)
        e2e = {"value": multirank.weak_scaling_value(cfg.tokens, world, 1, ems), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": ems, "steps": e_steps,
               "overlap": "H2D of step i+1 and D2H of step i-1 overlap the scan of step i "
                          "(two device buffer sets, three streams); pipeline fill and drain "
                          "inside the timed region"}

    if rank == 0:
        peaks, peak_src = load_peaks()
        ab = alg_bytes(cfg, es)
        af = alg_flops(cfg)
        dom = "bwd" if do_bwd else "fwd"
        dom_ms = bwd_ms if do_bwd else fwd_ms
        achieved = ab[dom] / (dom_ms * 1e-3) / 1e9
        traffic, tkernel = kernel_traffic(cfg, dom)
        step_bytes = ab["fwd"] + (ab["bwd"] if do_bwd else 0)
        step_flops = af["fwd"] + (af["bwd"] if do_bwd else 0)
        t_roof = max(step_bytes / (peaks["hbm_gbs"] * 1e9),
                     step_flops / (peaks["bf16_tflops"] * 1e12))
        ms_step = ms / args.steps
        line = {
            "metric": METRIC,
            "value": multirank.weak_scaling_value(cfg.tokens, world, args.steps, ms),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": cfg.dtype,
            "data": "synthetic (seeded generator; no dataset or trained weights)",
            "config": {"workload": cfg.name, "B": B, "H": H, "T": T, "d_in": di, "d_out": do,
                       "passes": "+".join(cfg.passes), "global_batch": multirank.global_batch(B, world),
                       "parallelism": f"independent batch per GPU x{world}" +
                                      (" + dW0 all-reduce" if world > 1 and do_bwd else ""),
                       "l2": "no flush: working set "
                             f"{step_bytes / 1e6:.0f} MB per step > 126 MB L2"},
            "roofline": {"bound": "hbm", "achieved": achieved,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                         "kernel": f"gradlev_scan_{dom} call (" +
                                   ("bwd kernel + dW0 reduce" if do_bwd else "fwd kernel") + ")",
                         "alg_bytes_per_launch": ab[dom], "ms_per_launch": dom_ms,
                         "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                                        if peak_src == "measured" else "fallback",
                         "step_frac_of_roofline": t_roof / (ms_step * 1e-3)},
            "breakdown": {"fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
                          "fwd_alg_bytes": ab["fwd"], "bwd_alg_bytes": ab["bwd"] if do_bwd else 0,
                          "alg_flops_per_step": step_flops,
                          "tflops": step_flops / (ms_step * 1e-3) / 1e12},
            "clocks": clk,
            "gpu_launches": gpu_launches,
            "e2e": e2e,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(cfg, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
