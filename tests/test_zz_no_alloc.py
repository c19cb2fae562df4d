"""gradlev_scan_bwd_noalloc: the reverse scan for callers that cannot allocate.

Callers such as fixed-pool serving runtimes, or plugins that are handed only
their tensors, cannot obtain a workspace. This entry point takes its scratch
from a static device array instead. The tests call it through the C ABI and
compare it with gradlev_scan_bwd (the entry point with a caller workspace).
Both run the same deterministic kernels, so the outputs must agree bit for bit,
on consecutive calls that share the array. The cases cover the CUDA-core
kernels (d = 64, bf16 and float32) and the tensor-core kernels (bf16, d_in =
128): a batch that fills the GPU, a small batch whose scans are cut into
segments, and d_out = 256. They also cover the status word the call leaves in
the array, and the launch count.

This file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest

import token_weight_scans_b200 as tw
from token_weight_scans_b200 import build as tw_build
from token_weight_scans_b200 import inputs
from tests.helpers import to_device, to_numpy

OUTS = ("dx", "dg", "deta", "dalpha", "dW0")
SCRATCH = 64 << 20


def _lib():
    tw_build.build()
    L = tw.lib()
    I, P, Z = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    L.gradlev_scan_bwd_noalloc.argtypes = [I] * 6 + [P] * 13
    L.gradlev_scan_bwd_noalloc.restype = I
    L.gradlev_scan_bwd_noalloc_scratch_bytes.argtypes = [I] * 7
    L.gradlev_scan_bwd_noalloc_scratch_bytes.restype = Z
    L.gradlev_noalloc_device_status.argtypes = [P]
    L.gradlev_noalloc_device_status.restype = I
    return L


def test_noalloc_scratch_query_and_limit():
    """Needs no GPU: the sizing is host arithmetic and the size check comes before any
    CUDA call."""
    L = _lib()
    P = ctypes.c_void_p
    need = L.gradlev_scan_bwd_noalloc_scratch_bytes
    # without checkpoints the need is the reverse scan's whole workspace
    for shape in ((8, 16, 4096, 128, 128, 1), (1, 16, 32768, 128, 256, 1), (2, 3, 300, 64, 64, 0)):
        assert need(*shape, 0) == L.gradlev_scan_workspace_bytes(*shape, 1)
        assert 0 < need(*shape, 1) < need(*shape, 0)
    # B8 H16 T4096 d128 without checkpoints needs ~1 GiB of states: rejected
    assert need(8, 16, 4096, 128, 128, 1, 0) > SCRATCH
    fake = P(4096)
    st = L.gradlev_scan_bwd_noalloc(8, 16, 4096, 128, 128, 1, *([fake] * 11), P(0), P(0))
    assert st == 3  # GRADLEV_ERR_WORKSPACE
    # with checkpoints only the partials are needed, which fit
    assert need(8, 16, 4096, 128, 128, 1, 1) <= SCRATCH
    assert need(8, 16, 4096, 130, 128, 1, 1) == 0  # unsupported shape (d_in % 4 != 0)


CASES = [
    # (dtype, B, H, T, d_in, d_out): CUDA-core kernels
    ("bf16", 2, 3, 300, 64, 64),
    ("f32", 2, 3, 300, 64, 64),
    # tensor-core kernels: one CTA per scan, every SM busy
    ("bf16", 8, 16, 512, 128, 128),
    # tensor-core kernels, few long scans: each scan is cut into segments
    ("bf16", 1, 2, 1024, 128, 128),
    ("bf16", 1, 2, 1024, 128, 256),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_noalloc_matches_bwd_bit_for_bit_on_consecutive_calls(case):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = _lib()
    dtype, B, H, T, di, do = case
    code = tw.BF16 if dtype == "bf16" else tw.F32
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    for call, (seed, use_ckpt) in enumerate(((31, False), (32, True), (33, False))):
        assert L.gradlev_scan_bwd_noalloc_scratch_bytes(B, H, T, di, do, code,
                                                        int(use_ckpt)) <= SCRATCH
        d = inputs.draw(B, H, T, di, do, dtype=dtype, alpha_mode="log_uniform", seed=seed)
        t = to_device(d, dtype)
        ck = None
        if use_ckpt:
            ck = torch.empty(tw.gradlev_scan_ckpt_bytes(B, H, T, di, do, code),
                             dtype=torch.uint8, device="cuda")
            tw.gradlev_scan_fwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], ckpt=ck)
        ref = tw.gradlev_scan_bwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], t["dy"],
                                  ckpt=ck)
        n_ref = tw.gradlev_last_launch_count()
        out = {k: torch.full_like(v, float("nan")) for k, v in ref.items()}
        P = lambda v: ctypes.c_void_p(v.data_ptr()) if v is not None else ctypes.c_void_p(0)
        st = L.gradlev_scan_bwd_noalloc(
            B, H, T, di, do, code, P(t["x"]), P(t["g"]), P(t["eta"]), P(t["alpha"]),
            P(t["W0"]), P(t["dy"]), P(out["dx"]), P(out["dg"]), P(out["deta"]),
            P(out["dalpha"]), P(out["dW0"]), P(ck), sp)
        assert st == 0, tw.gradlev_status_string(st)
        assert tw.gradlev_last_launch_count() == n_ref, "launch count of this call only"
        assert L.gradlev_noalloc_device_status(sp) == 0, "device-side wait timed out"
        torch.cuda.synchronize()
        for k in OUTS:
            a, b = to_numpy(out[k]), to_numpy(ref[k])
            assert np.all(np.isfinite(a)), (call, k)
            assert np.array_equal(a, b), (call, k, float(np.max(np.abs(a - b))))
