"""GPU tests of the deployment decode (gradlev_decode_step).

- **Parity.** y, the costates g and the carried deviation S after the call are
  compared against the float64 oracle's `decode` on the dtype-rounded inputs:
  - bf16 and f32;
  - d_in up to 128 (one float4 per lane) and up to 256 (two);
  - d_out not a multiple of the 16 rows of a CTA;
  - one token up to several dozen.
- **Token-by-token calls** must equal one call bit for bit: the same arithmetic
  runs in the same order.
- **Exact recovery on the GPU.** The tensor-core scan, driven by the decode's
  own costates and started from the same deviation, reproduces the decode's
  outputs and end state.
"""

import numpy as np
import pytest

import oracle
from token_weight_scans_b200 import inputs
from tests.helpers import TOL, rel_err, to_device, to_numpy

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


def _f64(d):
    return {k: v.astype(np.float64) for k, v in d.items()}


def start_state(B, H, din, dout, dtype, seed):
    """The deviation a previous 50-token decode left (realistic magnitude)."""
    pre = _f64(inputs.draw(B, H, 50, din, dout, dtype=dtype, alpha_mode="sigmoid", seed=seed,
                           with_v=True))
    _, _, S = oracle.decode(pre["x"], pre["v"], pre["eta"], pre["alpha"], pre["W0"],
                            np.zeros((B, H, dout, din)))
    return S.astype(np.float32)


CASES = [
    # (B, H, T, d_in, d_out, dtype)
    (2, 2, 1, 128, 128, "bf16"),
    (2, 2, 37, 128, 128, "bf16"),
    (2, 3, 20, 64, 48, "f32"),
    (1, 2, 5, 256, 100, "f32"),
    (1, 2, 9, 200, 33, "bf16"),
    (1, 1, 3, 4, 1, "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dT%d_%dx%d_%s" % c)
def test_decode_matches_oracle(case):
    import token_weight_scans_b200 as tw
    B, H, T, di, do, dt = case
    d = inputs.draw(B, H, T, di, do, dtype=dt, alpha_mode="sigmoid", seed=900 + T + di,
                    with_v=True)
    S0 = start_state(B, H, di, do, dt, seed=950 + T)
    t = to_device(d, dt)
    S = torch.from_numpy(S0).cuda()
    y, g = tw.gradlev_decode_step(t["x"], t["v"], t["eta"], t["alpha"], t["W0"], S)
    torch.cuda.synchronize()
    a = _f64(d)
    yr, gr, Sr = oracle.decode(a["x"], a["v"], a["eta"], a["alpha"], a["W0"],
                               S0.astype(np.float64))
    tol = TOL[dt]
    for name, got, ref in (("y", y, yr), ("g", g, gr), ("S", S, Sr)):
        err = rel_err(to_numpy(got), ref)
        assert err <= tol, (case, name, err)


def test_decode_token_by_token_equals_one_call():
    import token_weight_scans_b200 as tw
    B, H, T, di, do = 2, 2, 12, 128, 128
    d = inputs.draw(B, H, T, di, do, dtype="bf16", alpha_mode="sigmoid", seed=961, with_v=True)
    t = to_device(d, "bf16")
    S0 = torch.from_numpy(start_state(B, H, di, do, "bf16", seed=962)).cuda()
    S_all = S0.clone()
    y_all, g_all = tw.gradlev_decode_step(t["x"], t["v"], t["eta"], t["alpha"], t["W0"], S_all)
    S_one = S0.clone()
    ys, gs = [], []
    for k in range(T):
        sl = lambda a: a[:, :, k:k + 1].contiguous()
        yk, gk = tw.gradlev_decode_step(sl(t["x"]), sl(t["v"]), sl(t["eta"]), sl(t["alpha"]),
                                        t["W0"], S_one)
        ys.append(yk)
        gs.append(gk)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(ys, dim=2), y_all)
    assert torch.equal(torch.cat(gs, dim=2), g_all)
    assert torch.equal(S_one, S_all)


def test_scan_with_decode_costates_recovers_decode_on_gpu():
    import token_weight_scans_b200 as tw
    B, H, T, di, do = 2, 2, 150, 128, 128
    d = inputs.draw(B, H, T, di, do, dtype="bf16", alpha_mode="sigmoid", seed=971, with_v=True)
    t = to_device(d, "bf16")
    S0 = torch.from_numpy(start_state(B, H, di, do, "bf16", seed=972)).cuda()
    S = S0.clone()
    y, g = tw.gradlev_decode_step(t["x"], t["v"], t["eta"], t["alpha"], t["W0"], S)
    ys, ST = tw.gradlev_scan_fwd_state(t["x"], g, t["eta"], t["alpha"], t["W0"], S0)
    torch.cuda.synchronize()
    assert rel_err(to_numpy(ys), to_numpy(y)) <= TOL["bf16"]
    assert rel_err(to_numpy(ST), to_numpy(S)) <= TOL["bf16"]
