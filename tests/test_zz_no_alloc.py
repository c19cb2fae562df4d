"""gradlev_scan_bwd_noalloc: the reverse scan for callers that cannot allocate.

Callers such as fixed-pool serving runtimes or plugins that are handed only
their tensors cannot obtain a workspace; this entry point takes its scratch
from a static device array instead. These tests call it through the C ABI and
check it against gradlev_scan_bwd (the entry point with a caller workspace)
within the parity tolerance, on consecutive calls that share the array.

This file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest

import token_weight_scans_b200 as tw
from token_weight_scans_b200 import build as tw_build
from token_weight_scans_b200 import inputs
from tests.helpers import TOL, rel_err, to_device, to_numpy

OUTS = ("dx", "dg", "deta", "dalpha", "dW0")
SCRATCH = 64 << 20


def _fn():
    tw_build.build()
    L = tw.lib()
    f = L.gradlev_scan_bwd_noalloc
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 13
    f.restype = ctypes.c_int
    return f


def test_noalloc_rejects_problems_beyond_the_scratch():
    """Needs no GPU: the size check comes before any CUDA call."""
    f = _fn()
    P = ctypes.c_void_p
    fake = P(4096)
    # B8 H16 T4096 d128 without checkpoints needs ~1 GiB of states: rejected
    st = f(8, 16, 4096, 128, 128, 1, *([fake] * 11), P(0), P(0))
    assert st == 3  # GRADLEV_ERR_WORKSPACE
    # with checkpoints only the dW0 partials are needed: 8 MiB, accepted past the size check
    need = 256 + 8 * 16 * 128 * 128 * 4
    assert need <= SCRATCH


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_bwd_on_consecutive_calls(dtype):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    f = _fn()
    code = tw.BF16 if dtype == "bf16" else tw.F32
    B, H, T, di, do = 2, 3, 300, 64, 64
    stream = torch.cuda.current_stream()
    for call, (seed, use_ckpt) in enumerate(((31, False), (32, False), (33, True))):
        d = inputs.draw(B, H, T, di, do, dtype=dtype, alpha_mode="log_uniform", seed=seed)
        t = to_device(d, dtype)
        ck = None
        if use_ckpt:
            ck = torch.empty(tw.gradlev_scan_ckpt_bytes(B, H, T, di, do, code),
                             dtype=torch.uint8, device="cuda")
            tw.gradlev_scan_fwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], ckpt=ck)
        ref = tw.gradlev_scan_bwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], t["dy"])
        out = {k: torch.full_like(v, float("nan")) for k, v in ref.items()}
        P = lambda v: ctypes.c_void_p(v.data_ptr()) if v is not None else ctypes.c_void_p(0)
        st = f(B, H, T, di, do, code, P(t["x"]), P(t["g"]), P(t["eta"]), P(t["alpha"]),
               P(t["W0"]), P(t["dy"]), P(out["dx"]), P(out["dg"]), P(out["deta"]),
               P(out["dalpha"]), P(out["dW0"]), P(ck), ctypes.c_void_p(stream.cuda_stream))
        assert st == 0, tw.gradlev_status_string(st)
        torch.cuda.synchronize()
        for k in OUTS:
            a, b = to_numpy(out[k]), to_numpy(ref[k])
            assert np.all(np.isfinite(a)), (call, k)
            assert rel_err(a, b) <= TOL[dtype], (call, k, rel_err(a, b))
