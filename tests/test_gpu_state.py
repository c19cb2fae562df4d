"""GPU parity of the carried-state calls (a sequence split across calls).

gradlev_scan_fwd_state / gradlev_scan_bwd_state against the float64 oracle's
fwd_state / bwd_state:
- every output, S_T and dS_0 included;
- on the tensor-core path (d_out 128 and 256; a lone scan cut into segments,
  where the start state and the incoming adjoint enter the combine pass);
- on the CUDA-core path (bf16 and f32).

Two more checks:
- a split sequence chained on the GPU (S_T -> S_0 forward, dS_0 -> Lam_T in
  reverse) must match the oracle's whole sequence;
- the calls without a state must equal the plain calls bit for bit.

The start states and incoming adjoints are realistic magnitudes: the oracle's
S_T of an earlier seeded part and dS_0 of a later one.
"""

import numpy as np
import pytest

import oracle
from token_weight_scans_b200 import inputs
from tests.helpers import TOL, rel_err, to_device, to_numpy

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

OUTS = ("dx", "dg", "deta", "dalpha", "dW0", "dS0")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from token_weight_scans_b200 import build
    build.build()
    import token_weight_scans_b200 as tw
    tw.lib()
    yield


def _f64(d):
    return {k: v.astype(np.float64) for k, v in d.items()}


def carried(B, H, din, dout, dtype, seed):
    """(S0, LamT): the end state of an earlier part and the start adjoint of a later one."""
    pre = _f64(inputs.draw(B, H, 150, din, dout, dtype=dtype, alpha_mode="log_uniform",
                           seed=seed + 1))
    _, S0 = oracle.fwd_state(pre["x"], pre["g"], pre["eta"], pre["alpha"], pre["W0"])
    post = _f64(inputs.draw(B, H, 150, din, dout, dtype=dtype, alpha_mode="log_uniform",
                            seed=seed + 2))
    LamT = oracle.bwd_state(post["x"], post["g"], post["eta"], post["alpha"], post["W0"],
                            post["dy"])["dS0"]
    return S0.astype(np.float32), LamT.astype(np.float32)


def gpu_state(d, dtype, S0, LamT, use_ckpt=True):
    import token_weight_scans_b200 as tw
    t = to_device(d, dtype)
    B, H, T, di = t["x"].shape
    do = t["g"].shape[-1]
    code = tw.BF16 if dtype == "bf16" else tw.F32
    s0 = torch.from_numpy(S0).cuda() if S0 is not None else None
    lt = torch.from_numpy(LamT).cuda() if LamT is not None else None
    ws = torch.empty(tw.gradlev_scan_workspace_bytes(B, H, T, di, do, code, 1), dtype=torch.uint8,
                     device="cuda")
    ck = None
    if use_ckpt:
        ck = torch.empty(tw.gradlev_scan_ckpt_bytes(B, H, T, di, do, code), dtype=torch.uint8,
                         device="cuda")
    y, ST = tw.gradlev_scan_fwd_state(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], s0, ckpt=ck,
                                      workspace=ws)
    assert tw.gradlev_device_status(ws) == 0
    out = tw.gradlev_scan_bwd_state(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], t["dy"], s0,
                                    lt, ckpt=ck, workspace=ws)
    assert tw.gradlev_device_status(ws) == 0, "device-side wait timed out"
    res = {k: to_numpy(v) for k, v in out.items()}
    res["y"], res["ST"] = to_numpy(y), to_numpy(ST)
    return res


def oracle_state(d, S0, LamT):
    a = _f64(d)
    S0 = None if S0 is None else S0.astype(np.float64)
    LamT = None if LamT is None else LamT.astype(np.float64)
    y, ST = oracle.fwd_state(a["x"], a["g"], a["eta"], a["alpha"], a["W0"], S0)
    ref = oracle.bwd_state(a["x"], a["g"], a["eta"], a["alpha"], a["W0"], a["dy"], S0=S0,
                           LamT=LamT)
    ref["y"], ref["ST"] = y, ST
    return ref


def check(got, ref, tol, ctx):
    for k in ("y", "ST") + OUTS:
        err = rel_err(got[k], ref[k])
        assert err <= tol, (ctx, k, err)


CASES = [
    # (B, H, T, d_in, d_out, dtype): tensor-core path unsegmented (two chunks: the kernels
    # take S_0 / Lam_T and write S_T / dS_0 themselves) and segmented (the combine pass
    # takes them), its d_out = 256 slices, a lone scan cut into 8 segments, and the
    # CUDA-core path in both I/O types
    (2, 2, 100, 128, 128, "bf16"),
    (2, 2, 200, 128, 128, "bf16"),
    (1, 2, 130, 128, 256, "bf16"),
    (1, 2, 1000, 128, 128, "bf16"),
    (2, 2, 100, 64, 64, "bf16"),
    (2, 2, 77, 32, 48, "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dT%d_%dx%d_%s" % c)
def test_state_calls_match_oracle(case):
    B, H, T, di, do, dt = case
    d = inputs.draw(B, H, T, di, do, dtype=dt, alpha_mode="log_uniform", seed=700 + T)
    S0, LamT = carried(B, H, di, do, dt, seed=800 + T)
    check(gpu_state(d, dt, S0, LamT), oracle_state(d, S0, LamT), TOL[dt], case)


def test_state_bwd_without_checkpoints_starts_from_S0():
    d = inputs.draw(2, 2, 333, 128, 128, dtype="bf16", alpha_mode="log_uniform", seed=731)
    S0, LamT = carried(2, 2, 128, 128, "bf16", seed=732)
    check(gpu_state(d, "bf16", S0, LamT, use_ckpt=False), oracle_state(d, S0, LamT),
          TOL["bf16"], "own states")


@pytest.mark.parametrize("case", [(2, 2, 200, 128, 128, "bf16"), (2, 2, 77, 32, 48, "f32")],
                         ids=["tc", "ffma"])
def test_no_state_equals_plain_calls(case):
    import token_weight_scans_b200 as tw
    B, H, T, di, do, dt = case
    d = inputs.draw(B, H, T, di, do, dtype=dt, alpha_mode="log_uniform", seed=741)
    t = to_device(d, dt)
    y0 = tw.gradlev_scan_fwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"])
    o0 = tw.gradlev_scan_bwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], t["dy"])
    y1, _ = tw.gradlev_scan_fwd_state(t["x"], t["g"], t["eta"], t["alpha"], t["W0"])
    o1 = tw.gradlev_scan_bwd_state(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], t["dy"])
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    for k in o0:
        assert torch.equal(o0[k], o1[k]), k


@pytest.mark.parametrize("split", [64, 100])
def test_split_sequence_chained_on_gpu(split):
    """Two calls per direction, chained through S_T -> S_0 and dS_0 -> Lam_T on the GPU,
    reproduce the oracle's whole sequence."""
    import token_weight_scans_b200 as tw
    B, H, T = 2, 2, 260
    d = inputs.draw(B, H, T, 128, 128, dtype="bf16", alpha_mode="log_uniform", seed=751)
    ref = oracle_state(d, None, None)
    t = to_device(d, "bf16")
    part = lambda t0, t1: {k: (v[:, :, t0:t1].contiguous() if k != "W0" else v)
                           for k, v in t.items()}
    a, b = part(0, split), part(split, T)
    ya, Sa = tw.gradlev_scan_fwd_state(a["x"], a["g"], a["eta"], a["alpha"], a["W0"])
    yb, Sb = tw.gradlev_scan_fwd_state(b["x"], b["g"], b["eta"], b["alpha"], b["W0"], Sa)
    ob = tw.gradlev_scan_bwd_state(b["x"], b["g"], b["eta"], b["alpha"], b["W0"], b["dy"], Sa)
    oa = tw.gradlev_scan_bwd_state(a["x"], a["g"], a["eta"], a["alpha"], a["W0"], a["dy"],
                                   None, ob["dS0"])
    torch.cuda.synchronize()
    got = {"y": to_numpy(torch.cat([ya, yb], dim=2)), "ST": to_numpy(Sb)}
    for k in ("dx", "dg", "deta", "dalpha"):
        got[k] = to_numpy(torch.cat([oa[k], ob[k]], dim=2))
    got["dW0"] = to_numpy(oa["dW0"] + ob["dW0"])
    got["dS0"] = to_numpy(oa["dS0"])
    check(got, ref, TOL["bf16"], ("split", split))
