"""GPU tests of the consistency step (gradlev_consistency_step).

The step has four parts: the forward scan on predicted costates ghat, the
reconstructed costates gtil = y - v, the per-token token and consistency
losses, and every gradient of their sum. It is compared against the float64
oracle's `consistency`:
- on the tensor-core path (d_out 128 and 256) and the CUDA-core path (bf16, f32);
- with ghat the serial learner's true costates plus noise, so the residual is
  neither zero nor dominant.

At the fixed point (ghat = the serial costates) the consistency loss must
collapse to the rounding level of the I/O dtype.
"""

import numpy as np
import pytest

import oracle
from token_weight_scans_b200 import inputs
from tests.helpers import TOL, rel_err, to_device, to_numpy

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

OUTS = ("y", "gtil", "loss_tok", "loss_c", "dx", "dghat", "deta", "dalpha", "dW0", "dv")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from token_weight_scans_b200 import build
    build.build()
    import token_weight_scans_b200 as tw
    tw.lib()
    yield


def _case(B, H, T, di, do, dt, seed, noise):
    d = inputs.draw(B, H, T, di, do, dtype=dt, alpha_mode="sigmoid", seed=seed, with_v=True)
    a = {k: v.astype(np.float64) for k, v in d.items()}
    _, gstar = oracle.serial(a["x"], a["v"], a["eta"], a["alpha"], a["W0"])
    rng = np.random.default_rng(seed + 1)
    ghat = gstar + noise * np.std(gstar) * rng.standard_normal(gstar.shape)
    ghat = ghat.astype(np.float32)
    if dt == "bf16":
        ghat = inputs.round_bf16(ghat)
    return d, ghat


def _run(d, ghat, dt, lam):
    import token_weight_scans_b200 as tw
    t = to_device(d, dt)
    gh = torch.from_numpy(ghat).to(t["x"].dtype).cuda()
    out = tw.gradlev_consistency_step(t["x"], gh, t["eta"], t["alpha"], t["W0"], t["v"], lam)
    torch.cuda.synchronize()
    return {k: to_numpy(v) for k, v in out.items()}


CASES = [
    (2, 2, 200, 128, 128, "bf16"),
    (1, 2, 130, 128, 256, "bf16"),
    (2, 2, 100, 64, 64, "bf16"),
    (2, 2, 77, 32, 48, "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dT%d_%dx%d_%s" % c)
def test_consistency_step_matches_oracle(case):
    B, H, T, di, do, dt = case
    d, ghat = _case(B, H, T, di, do, dt, seed=1100 + T, noise=0.5)
    lam = 0.5
    got = _run(d, ghat, dt, lam)
    a = {k: v.astype(np.float64) for k, v in d.items()}
    ref = oracle.consistency(a["x"], ghat.astype(np.float64), a["eta"], a["alpha"], a["W0"],
                             a["v"], lam=lam)
    for k in OUTS:
        err = rel_err(got[k], ref[k])
        assert err <= TOL[dt], (case, k, err)


def test_consistency_loss_collapses_at_the_serial_costates():
    B, H, T, di, do = 2, 2, 300, 128, 128
    d, gstar = _case(B, H, T, di, do, "bf16", seed=1201, noise=0.0)
    _, ghat = _case(B, H, T, di, do, "bf16", seed=1201, noise=0.3)
    at = _run(d, gstar, "bf16", 1.0)
    off = _run(d, ghat, "bf16", 1.0)
    scale = np.sum(gstar.astype(np.float64) ** 2)
    assert np.sum(at["loss_c"]) < 1e-3 * scale
    assert np.sum(off["loss_c"]) > 1e-2 * scale
