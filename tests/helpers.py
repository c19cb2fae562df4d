"""Shared helpers of the parity tests (no scan arithmetic here)."""

import numpy as np

# Max-norm relative error bars (max |gpu - ref| / max |ref| per output tensor,
# against the float64 oracle run on the dtype-rounded inputs).
TOL = {"f32": 1e-5, "bf16": 2e-2}


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.max(np.abs(b)) if b.size else 0.0
    if den == 0.0:
        return float(np.max(np.abs(a))) if a.size else 0.0
    return float(np.max(np.abs(a - b)) / den)


def to_device(d, dtype, device="cuda"):
    """Upload a generator dict: x, g, dy (and v) in the I/O dtype, eta/alpha/W0 float32."""
    import torch
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = {}
    for k, v in d.items():
        t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
        if k in ("x", "g", "dy", "v"):
            t = t.to(tdt)
        out[k] = t.to(device)
    return out


def to_numpy(t):
    import torch
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def heads_slice(d, b, h):
    """Inputs of one (b, h) scan as a B = H = 1 problem (float64)."""
    out = {}
    for k, v in d.items():
        if k == "W0":
            out[k] = v[h:h + 1].astype(np.float64)
        else:
            out[k] = v[b:b + 1, h:h + 1].astype(np.float64)
    return out
