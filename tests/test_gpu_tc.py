"""GPU tests of the tensor-core (tcgen05) path: bf16, d_in = 128, d_out = 128 / 256.

Parity against the float64 oracle (max-norm relative error <= 2e-2 for bf16),
ragged lengths around the 64-token chunk, degenerate gates, bit-exact integer
inputs, determinism, and the bounded-wait failure path (a completion signal
that is withheld on purpose: the kernel must report GRADLEV_ERR_TIMEOUT and
leave the context usable; no fault, trap or hang is involved).
"""

import numpy as np
import pytest

import oracle
from token_weight_scans_b200 import inputs
from tests.helpers import TOL, heads_slice, rel_err, to_device, to_numpy

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from token_weight_scans_b200 import build
    build.build()
    import token_weight_scans_b200 as tw
    tw.lib()
    yield


def gpu_fwd(d):
    import token_weight_scans_b200 as tw
    t = to_device(d, "bf16")
    B, H, T, di = t["x"].shape
    ws = torch.empty(tw.gradlev_scan_workspace_bytes(B, H, T, di, t["g"].shape[-1], tw.BF16, 0),
                     dtype=torch.uint8, device="cuda")
    y = tw.gradlev_scan_fwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], workspace=ws)
    assert tw.gradlev_device_status(ws) == 0, "device-side wait timed out"
    return to_numpy(y)


def oracle_fwd(d):
    d64 = {k: v.astype(np.float64) for k, v in d.items()}
    return oracle.fwd(d64["x"], d64["g"], d64["eta"], d64["alpha"], d64["W0"])


@pytest.mark.parametrize("T", [1, 5, 63, 64, 65, 129, 300])
def test_tc_fwd_ragged_lengths(T):
    d = inputs.draw(2, 2, T, 128, 128, dtype="bf16", alpha_mode="log_uniform", seed=300 + T)
    err = rel_err(gpu_fwd(d), oracle_fwd(d))
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("mode", ["sigmoid", "log_uniform"])
def test_tc_fwd_several_chunks(mode):
    d = inputs.draw(3, 2, 1000, 128, 128, dtype="bf16", alpha_mode=mode, seed=41)
    err = rel_err(gpu_fwd(d), oracle_fwd(d))
    assert err <= TOL["bf16"], err


def test_tc_fwd_degenerate_gates():
    d = inputs.draw(2, 2, 200, 128, 128, dtype="bf16", seed=42)
    d["alpha"][..., ::9] = 0.0
    d["alpha"][..., 4::9] = 1.0
    d["eta"][..., 7::13] = 0.0
    err = rel_err(gpu_fwd(d), oracle_fwd(d))
    assert err <= TOL["bf16"], err


def test_tc_fwd_bit_exact_integer_inputs():
    """alpha = 1, eta = 1/8, sparse {-1,0,1} inputs: every product, sum, mask value and
    bf16 operand is exactly representable, so the result equals the oracle bit for bit."""
    rng = np.random.default_rng(3)
    B, H, T, di, do = 1, 2, 150, 128, 128
    sp = lambda *s, p=0.03: (rng.integers(-1, 2, s) * (rng.random(s) < p)).astype(np.float32)
    d = {"x": sp(B, H, T, di), "g": sp(B, H, T, do, p=0.05),
         "eta": np.full((B, H, T), 0.125, np.float32), "alpha": np.ones((B, H, T), np.float32),
         "W0": sp(H, do, di, p=0.05), "dy": sp(B, H, T, do)}
    ref = oracle_fwd(d)
    assert np.array_equal(inputs.round_bf16(ref).astype(np.float64), ref)
    got = gpu_fwd(d)
    assert np.array_equal(got, ref), rel_err(got, ref)


def test_tc_fwd_deterministic():
    d = inputs.draw(2, 3, 333, 128, 128, dtype="bf16", alpha_mode="log_uniform", seed=43)
    assert np.array_equal(gpu_fwd(d), gpu_fwd(d))


def test_tc_fwd_timeout_path_reports_and_recovers():
    import token_weight_scans_b200 as tw
    d = inputs.draw(2, 2, 256, 128, 128, dtype="bf16", seed=44)
    t = to_device(d, "bf16")
    ws = torch.zeros(tw.gradlev_scan_workspace_bytes(2, 2, 256, 128, 128, tw.BF16, 0),
                     dtype=torch.uint8, device="cuda")
    tw.lib().gradlev_debug_inject_timeout(1, 20)
    tw.gradlev_scan_fwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], workspace=ws)
    assert tw.gradlev_device_status(ws) == 5  # GRADLEV_ERR_TIMEOUT
    # the context is intact: a normal call right after succeeds and is correct
    y = tw.gradlev_scan_fwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], workspace=ws)
    assert tw.gradlev_device_status(ws) == 0
    assert rel_err(to_numpy(y), oracle_fwd(d)) <= TOL["bf16"]


# ------------------------------------------------------------------ reverse scan

BWD_OUTS = ("dx", "dg", "deta", "dalpha", "dW0")


def gpu_fwd_bwd(d, use_ckpt=True):
    import token_weight_scans_b200 as tw
    t = to_device(d, "bf16")
    B, H, T, di = t["x"].shape
    do = t["g"].shape[-1]
    ws = torch.empty(tw.gradlev_scan_workspace_bytes(B, H, T, di, do, tw.BF16, 1),
                     dtype=torch.uint8, device="cuda")
    ck = None
    if use_ckpt:
        ck = torch.empty(tw.gradlev_scan_ckpt_bytes(B, H, T, di, do, tw.BF16), dtype=torch.uint8,
                         device="cuda")
    y = tw.gradlev_scan_fwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], ckpt=ck, workspace=ws)
    assert tw.gradlev_device_status(ws) == 0
    out = tw.gradlev_scan_bwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], t["dy"], ckpt=ck,
                              workspace=ws)
    assert tw.gradlev_device_status(ws) == 0, "device-side wait timed out"
    res = {k: to_numpy(v) for k, v in out.items()}
    res["y"] = to_numpy(y)
    return res


def oracle_fwd_bwd(d):
    d64 = {k: v.astype(np.float64) for k, v in d.items()}
    o = oracle.bwd(d64["x"], d64["g"], d64["eta"], d64["alpha"], d64["W0"], d64["dy"])
    o["y"] = oracle.fwd(d64["x"], d64["g"], d64["eta"], d64["alpha"], d64["W0"])
    return o


def check_all(got, ref, ctx):
    errs = {k: rel_err(got[k], ref[k]) for k in ("y",) + BWD_OUTS}
    bad = {k: e for k, e in errs.items() if not e <= TOL["bf16"]}
    assert not bad, f"{ctx}: {errs}"


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 128, 200])
def test_tc_bwd_ragged_lengths(T):
    d = inputs.draw(2, 2, T, 128, 128, dtype="bf16", alpha_mode="log_uniform", seed=500 + T)
    check_all(gpu_fwd_bwd(d), oracle_fwd_bwd(d), f"T={T}")


@pytest.mark.parametrize("mode", ["sigmoid", "log_uniform"])
def test_tc_bwd_several_chunks(mode):
    d = inputs.draw(3, 2, 700, 128, 128, dtype="bf16", alpha_mode=mode, seed=51)
    check_all(gpu_fwd_bwd(d), oracle_fwd_bwd(d), mode)


def test_tc_bwd_degenerate_gates():
    d = inputs.draw(2, 2, 300, 128, 128, dtype="bf16", seed=52)
    d["alpha"][..., ::9] = 0.0
    d["alpha"][..., 4::9] = 1.0
    d["eta"][..., 7::13] = 0.0
    check_all(gpu_fwd_bwd(d), oracle_fwd_bwd(d), "degenerate gates")


def test_tc_bwd_own_state_sweep_matches_checkpoints():
    d = inputs.draw(2, 2, 333, 128, 128, dtype="bf16", alpha_mode="log_uniform", seed=53)
    a = gpu_fwd_bwd(d, use_ckpt=True)
    b = gpu_fwd_bwd(d, use_ckpt=False)
    for k in BWD_OUTS:
        assert np.array_equal(a[k], b[k]), k


def test_tc_bwd_deterministic():
    d = inputs.draw(2, 3, 260, 128, 128, dtype="bf16", alpha_mode="log_uniform", seed=54)
    a = gpu_fwd_bwd(d)
    b = gpu_fwd_bwd(d)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_tc_bwd_bit_exact_integer_inputs():
    rng = np.random.default_rng(5)
    B, H, T, di, do = 2, 2, 150, 128, 128
    sp = lambda *s, p=0.03: (rng.integers(-1, 2, s) * (rng.random(s) < p)).astype(np.float32)
    d = {"x": sp(B, H, T, di), "g": sp(B, H, T, do, p=0.05),
         "eta": np.full((B, H, T), 0.125, np.float32), "alpha": np.ones((B, H, T), np.float32),
         "W0": sp(H, do, di, p=0.05), "dy": sp(B, H, T, do, p=0.05)}
    ref = oracle_fwd_bwd(d)
    for k in ("y", "dx", "dg"):
        assert np.array_equal(inputs.round_bf16(ref[k]).astype(np.float64), ref[k]), k
    got = gpu_fwd_bwd(d)
    for k in ("y",) + BWD_OUTS:
        assert np.array_equal(got[k], ref[k]), (k, rel_err(got[k], ref[k]))


@pytest.mark.parametrize("T", [70, 200])
def test_tc_rectangular_dout256(T):
    """d_out = 256: forward on two 128-row slices, backward as two slice problems."""
    d = inputs.draw(2, 2, T, 128, 256, dtype="bf16", alpha_mode="log_uniform", seed=600 + T)
    check_all(gpu_fwd_bwd(d), oracle_fwd_bwd(d), f"d_out=256 T={T}")


def test_tc_segmented_scan_matches_unsegmented():
    """A lone scan is cut into segments walked by separate CTAs (summary, combine and
    main passes); the same scan as head 0 of a batch that fills the GPU runs in one
    segment. Both must agree to within the bf16 rounding of the outputs."""
    H, T = 80, 1000
    big = inputs.draw(1, H, T, 128, 128, dtype="bf16", alpha_mode="log_uniform", seed=61)
    lone = {k: (v[:, :1] if v.ndim >= 3 and k != "W0" else v[:1]) for k, v in big.items()}
    a = gpu_fwd_bwd(lone)
    b = gpu_fwd_bwd(big)
    for k in ("y", "dx", "dg", "deta", "dalpha"):
        err = rel_err(a[k], b[k][:, :1])
        assert err <= 1e-2, (k, err)
    assert rel_err(a["dW0"], b["dW0"][:1]) <= 1e-2
    ref = oracle_fwd_bwd(lone)
    check_all(a, ref, "segmented lone scan")


@pytest.fixture
def summary_rescale():
    """Sets the bound of the summary passes' deferred decay; restores the default after."""
    import token_weight_scans_b200 as tw
    yield tw.lib().gradlev_debug_summary_rescale
    tw.lib().gradlev_debug_summary_rescale(-1.0)


@pytest.mark.parametrize("dout", [128, 256])
@pytest.mark.parametrize("bound", [64.0, 4.0, 0.0],
                         ids=["default", "every-few-chunks", "every-chunk"])
def test_tc_segment_summary_deferred_decay(bound, dout, summary_rescale):
    """The summary passes keep the decay since the last in-place rescale of the carried
    matrix as a scale 2^E outside tensor memory and rescale the matrix once E would drop
    below -bound. Sixteen scans of 72 chunks are cut into 9 segments of 8 chunks; the
    same scans run unsegmented as heads of a batch of 80 (no summary pass). With these
    gates (about -1.3 of log2 decay per chunk) the rescale never runs at the default
    bound, every few chunks at 4 and at every chunk at 0; the results agree with the
    unsegmented run and with the oracle whatever the bound. At d_out = 256 the reverse's
    summary pass carries both 128-row slices of the adjoint in one CTA."""
    summary_rescale(bound)
    H, T = 80, 72 * 64
    big = inputs.draw(1, H, T, 128, dout, dtype="bf16", alpha_mode="log_uniform", seed=62)
    lone = {k: (v[:16] if k == "W0" else v[:, :16]) for k, v in big.items()}
    a = gpu_fwd_bwd(lone)
    b = gpu_fwd_bwd(big)
    for k in ("y", "dx", "dg", "deta", "dalpha"):
        err = rel_err(a[k], b[k][:, :16])
        assert err <= 1e-2, (k, err)
    assert rel_err(a["dW0"], b["dW0"][:16]) <= 1e-2
    got = {k: (a[k][5:6] if k == "dW0" else a[k][:, 5:6]) for k in ("y",) + BWD_OUTS}
    check_all(got, oracle_fwd_bwd(heads_slice(lone, 0, 5)), f"segmented, bound {bound}, d_out {dout}")


# ------------------------------------------------------------------ bounded-wait failure path
# Each site of the test hook withholds one completion signal of one kernel family: the
# kernel's bounded wait runs out, every CTA unwinds, the device status reports
# GRADLEV_ERR_TIMEOUT, and the next call on the same context is correct. No fault, trap
# or hang is involved.

TIMEOUT = 5  # GRADLEV_ERR_TIMEOUT


def _timeout_then_recover(site, B, H, T):
    import token_weight_scans_b200 as tw
    d = inputs.draw(B, H, T, 128, 128, dtype="bf16", alpha_mode="log_uniform", seed=70 + site)
    t = to_device(d, "bf16")
    ws = torch.zeros(tw.gradlev_scan_workspace_bytes(B, H, T, 128, 128, tw.BF16, 1),
                     dtype=torch.uint8, device="cuda")
    ck = torch.empty(tw.gradlev_scan_ckpt_bytes(B, H, T, 128, 128, tw.BF16), dtype=torch.uint8,
                     device="cuda")
    fwd = lambda: tw.gradlev_scan_fwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], ckpt=ck,
                                      workspace=ws)
    bwd = lambda: tw.gradlev_scan_bwd(t["x"], t["g"], t["eta"], t["alpha"], t["W0"], t["dy"],
                                      ckpt=ck, workspace=ws)
    if site in (2, 4):  # the reverse scan needs good checkpoints first
        fwd()
        assert tw.gradlev_device_status(ws) == 0
    tw.lib().gradlev_debug_inject_timeout(site, 20)
    fwd() if site in (1, 3) else bwd()
    assert tw.gradlev_device_status(ws) == TIMEOUT
    # the context is intact: normal calls right after succeed and are correct
    y = fwd()
    assert tw.gradlev_device_status(ws) == 0
    out = bwd()
    assert tw.gradlev_device_status(ws) == 0
    got = {k: to_numpy(v) for k, v in out.items()}
    got["y"] = to_numpy(y)
    check_all(got, oracle_fwd_bwd(d), f"after a timeout at site {site}")


def test_tc_bwd_timeout_path_reports_and_recovers():
    _timeout_then_recover(2, 2, 2, 256)


@pytest.mark.parametrize("site", [3, 4], ids=["fwd-summary", "bwd-summary"])
def test_tc_segment_summary_timeout_reports_and_recovers(site):
    import token_weight_scans_b200 as tw
    # one lone long scan: cut into segments, so the summary passes run
    assert tw.gradlev_scan_workspace_bytes(1, 1, 1024, 128, 128, tw.BF16, 0) > 256
    _timeout_then_recover(site, 1, 1, 1024)
