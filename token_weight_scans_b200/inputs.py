"""Seeded synthetic inputs for the GradLev scan.

This module draws random numbers and rounds them to the storage dtype; it
contains none of the scan's arithmetic. Both the CUDA path (tests, bench,
smoke) and the float64 oracle consume exactly the arrays it returns.

Recipe (fixed draw order x, g, eta_raw, alpha_raw, W0, dy, v; all draws in
float64 from numpy's PCG64 with the given seed, then rounded):

* x ~ N(0, 1/d_in), g ~ N(0, 1), dy ~ N(0, 1), v ~ N(0, 1)
* eta = 0.1 * sigmoid(N(0, 1))
* alpha = 0.9 + 0.1 * sigmoid(N(0, 1))        (``alpha_mode="sigmoid"``)
  alpha = 1 - 10**U(-4, -1)                    (``alpha_mode="log_uniform"``)
* W0 ~ N(0, 1/d_in), one matrix per head, float32
* x, g, dy (and v) are rounded to the I/O dtype (bf16 round-to-nearest-even or
  fp32); eta, alpha and W0 are always float32.

All arrays are returned as float32 numpy arrays whose values are exactly
representable in the I/O dtype, so the oracle can upcast them to float64
without further rounding.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

SEED_BASE = 20261202


@dataclass(frozen=True)
class ScanConfig:
    name: str
    B: int
    H: int
    T: int
    d_in: int
    d_out: int
    dtype: str            # "f32" or "bf16": dtype of x, g, y, dy, dx, dg
    alpha_mode: str       # "sigmoid" or "log_uniform"
    passes: tuple = ("fwd", "bwd")
    index: int = -1

    @property
    def head_tokens(self) -> int:
        return self.B * self.H * self.T

    @property
    def tokens(self) -> int:
        return self.B * self.T


# The five workloads of the method's scan: a tiny float64 check, an fp32 scan,
# the bf16 forward, the bf16 forward+backward and the long-context rectangular
# case. Config 0 is run by the GPU on its fp32 path.
CONFIGS = [
    ScanConfig("tiny_f64_B1H1T256d16", 1, 1, 256, 16, 16, "f32", "sigmoid", ("fwd", "bwd"), 0),
    ScanConfig("f32_B4H8T2048d64", 4, 8, 2048, 64, 64, "f32", "sigmoid", ("fwd", "bwd"), 1),
    ScanConfig("bf16_fwd_B8H16T4096d128", 8, 16, 4096, 128, 128, "bf16", "sigmoid", ("fwd",), 2),
    ScanConfig("bf16_fwdbwd_B8H16T4096d128", 8, 16, 4096, 128, 128, "bf16", "log_uniform",
               ("fwd", "bwd"), 3),
    ScanConfig("bf16_long_B1H16T32768din128dout256", 1, 16, 32768, 128, 256, "bf16",
               "log_uniform", ("fwd", "bwd"), 4),
]


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float values to the nearest bfloat16 (ties to even); returns float32."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(f)
    out = r.astype(np.uint32).view(np.float32).copy()
    out[nan] = np.nan
    return out


def _round(a: np.ndarray, dtype: str) -> np.ndarray:
    a = np.asarray(a, dtype=np.float32)
    if dtype == "bf16":
        return round_bf16(a)
    if dtype == "f32":
        return np.ascontiguousarray(a)
    raise ValueError(f"unknown dtype {dtype!r}")


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def draw(B: int, H: int, T: int, d_in: int, d_out: int, *, dtype: str = "f32",
         alpha_mode: str = "sigmoid", seed: int = SEED_BASE, with_v: bool = False) -> dict:
    """Draw one seeded input set (see the module docstring for the recipe)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}
    out["x"] = _round(rng.standard_normal((B, H, T, d_in)) / np.sqrt(d_in), dtype)
    out["g"] = _round(rng.standard_normal((B, H, T, d_out)), dtype)
    out["eta"] = (0.1 * _sigmoid(rng.standard_normal((B, H, T)))).astype(np.float32)
    if alpha_mode == "sigmoid":
        out["alpha"] = (0.9 + 0.1 * _sigmoid(rng.standard_normal((B, H, T)))).astype(np.float32)
    elif alpha_mode == "log_uniform":
        out["alpha"] = (1.0 - 10.0 ** rng.uniform(-4.0, -1.0, (B, H, T))).astype(np.float32)
    else:
        raise ValueError(f"unknown alpha_mode {alpha_mode!r}")
    out["W0"] = (rng.standard_normal((H, d_out, d_in)) / np.sqrt(d_in)).astype(np.float32)
    out["dy"] = _round(rng.standard_normal((B, H, T, d_out)), dtype)
    if with_v:
        out["v"] = _round(rng.standard_normal((B, H, T, d_out)), dtype)
    return out


def draw_config(cfg: ScanConfig, *, with_v: bool = False, seed=None) -> dict:
    """Draw the inputs of one named workload with its own seed (SEED_BASE + index)."""
    s = SEED_BASE + max(cfg.index, 0) if seed is None else seed
    return draw(cfg.B, cfg.H, cfg.T, cfg.d_in, cfg.d_out, dtype=cfg.dtype,
                alpha_mode=cfg.alpha_mode, seed=s, with_v=with_v)
