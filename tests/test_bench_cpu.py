"""CPU checks of bench.py's contract: the reference arm's JSON line, the other ranks'
silence in that arm, and the algorithmic byte counts behind the roofline object."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT,
                          env=env, capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_the_contract_line():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "0", "--config", "0"])
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["value"] > 0 and line["unit"] == "tokens/s" and line["higher_is_better"]
    assert line["config"]["workload"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert cb["sample"]
    e = line["e2e"]
    assert e["value"] == line["value"] and e["unit"] == line["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "0", "--config", "0"],
             env_extra={"RANK": "1", "WORLD_SIZE": "2"}, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_algorithmic_bytes_match_the_stated_per_unit_figures():
    """The roofline's bytes: every input read once, every output written once. For the
    bf16 d = 128 workload that is 776 B (fwd) and 1296 B (bwd) per head-token, plus W0 (and
    dW0) once per head."""
    sys.path.insert(0, ROOT)
    import bench
    from token_weight_scans_b200 import inputs
    cfg = inputs.CONFIGS[3]
    N = cfg.B * cfg.H * cfg.T
    w = cfg.H * cfg.d_in * cfg.d_out * 4
    ab = bench.alg_bytes(cfg, 2)
    assert ab["fwd"] == N * 776 + w
    assert ab["bwd"] == N * 1296 + 2 * w
    assert ab["bwd"] == pytest.approx(681.6e6, rel=1e-3)


def test_traffic_record_applies_to_its_call_and_workload_only():
    """The committed DRAM-traffic record is reported only for the call and workload it was
    taken on, and only while the kernel source is the one it was taken from."""
    import dataclasses
    import hashlib
    sys.path.insert(0, ROOT)
    import bench
    from token_weight_scans_b200 import inputs
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)
    src = open(os.path.join(ROOT, rec["source"]), "rb").read()
    current = hashlib.sha256(src).hexdigest() == rec["source_sha256"]
    w = rec["workload"]
    match = [c for c in inputs.CONFIGS
             if {"B": c.B, "H": c.H, "T": c.T, "d_in": c.d_in, "d_out": c.d_out} == w]
    assert match, "the record names a workload that no configuration has"
    cfg = match[0]
    got, kernel = bench.kernel_traffic(cfg, rec["call"])
    assert kernel == rec["kernel"]
    assert got == (rec["bytes_per_launch"] if current else None)
    other = "fwd" if rec["call"] == "bwd" else "bwd"
    assert bench.kernel_traffic(cfg, other)[0] is None
    reduced = dataclasses.replace(cfg, B=cfg.B // 2)
    assert bench.kernel_traffic(reduced, rec["call"])[0] is None
