"""GPU tests of the two-layer reconstruction (gradlev_mlp2_recon).

The two-layer adapted MLP is the pages' synthetic test. Its outputs, a, h, y,
the reconstructed costates and the first-matrix gradient, are compared against
the float64 oracle:
- on tensor-core scan shapes (d = 128) and on the CUDA-core path (bf16 and f32);
- with given costates equal to the serial learner's plus noise.

The mechanism itself is then checked on the GPU: with the serial learner's
costates supplied, the reconstruction gives them back to the I/O dtype's
rounding, while the control (persistent second matrix) does not.
"""

import numpy as np
import pytest

import oracle
from token_weight_scans_b200 import inputs
from tests.helpers import TOL, rel_err, to_numpy

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


def draw(B, H, T, dx, dh, dy, dt, seed):
    """Seeded inputs, scaled so that tanh is not saturated and the adaptation stays bounded;
    the dtype's rounding is applied before either side sees them."""
    rng = np.random.default_rng(seed)
    rnd = inputs.round_bf16 if dt == "bf16" else (lambda a: a)
    f = lambda a: rnd(a.astype(np.float32))
    d = dict(x=f(rng.standard_normal((B, H, T, dx))), v=f(rng.standard_normal((B, H, T, dy))),
             eta=(1.0 / dx * rng.random((B, H, T))).astype(np.float32),
             alpha=rng.uniform(0.9, 0.999, (B, H, T)).astype(np.float32),
             W1=(rng.standard_normal((H, dh, dx)) / np.sqrt(dx)).astype(np.float32),
             W2=(rng.standard_normal((H, dy, dh)) / np.sqrt(dh)).astype(np.float32))
    a64 = {k: v.astype(np.float64) for k, v in d.items()}
    _, g1, g2 = oracle.mlp2_serial(a64["x"], a64["v"], a64["eta"], a64["alpha"], a64["W1"],
                                   a64["W2"])
    return d, f(g1), f(g2), rng


def gpu(d, g1, g2, dt, control=False):
    import token_weight_scans_b200 as tw
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    t = {k: torch.from_numpy(v).cuda() for k, v in d.items()}
    for k in ("x", "v"):
        t[k] = t[k].to(tdt)
    out = tw.gradlev_mlp2_recon(t["x"], torch.from_numpy(g1).to(tdt).cuda(),
                                torch.from_numpy(g2).to(tdt).cuda(), t["v"], t["eta"],
                                t["alpha"], t["W1"], t["W2"], control)
    torch.cuda.synchronize()
    return {k: to_numpy(v) for k, v in out.items()}


def ref(d, g1, g2, control=False):
    a = {k: v.astype(np.float64) for k, v in d.items()}
    return oracle.mlp2_recon(a["x"], g1.astype(np.float64), g2.astype(np.float64), a["v"],
                             a["eta"], a["alpha"], a["W1"], a["W2"], control=control)


CASES = [
    # (B, H, T, d_x, d_h, d_y, dtype)
    (2, 2, 200, 128, 128, 128, "bf16"),
    (1, 2, 100, 64, 64, 64, "bf16"),
    (2, 2, 77, 32, 48, 16, "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dT%d_%dx%dx%d_%s" % c)
@pytest.mark.parametrize("control", [False, True], ids=["adapted", "control"])
def test_mlp2_recon_matches_oracle(case, control):
    B, H, T, dx, dh, dy, dt = case
    d, g1, g2, rng = draw(B, H, T, dx, dh, dy, dt, seed=1300 + T)
    noise = lambda g: (g + 0.3 * np.std(g) * rng.standard_normal(g.shape)).astype(np.float32)
    rnd = inputs.round_bf16 if dt == "bf16" else (lambda a: a)
    g1n, g2n = rnd(noise(g1)), rnd(noise(g2))
    got, want = gpu(d, g1n, g2n, dt, control), ref(d, g1n, g2n, control)
    for k in ("a", "h", "y", "g2til", "g1til", "dW1"):
        err = rel_err(got[k], want[k])
        assert err <= TOL[dt], (case, control, k, err)


def test_mlp2_exact_recovery_and_control_on_gpu():
    B, H, T, dx, dh, dy = 2, 2, 256, 128, 128, 128
    d, g1, g2, _ = draw(B, H, T, dx, dh, dy, "bf16", seed=1401)
    got = gpu(d, g1, g2, "bf16")
    ctl = gpu(d, g1, g2, "bf16", control=True)
    assert rel_err(got["g1til"], g1) <= TOL["bf16"]
    assert rel_err(got["g2til"], g2) <= TOL["bf16"]
    assert np.array_equal(ctl["y"], got["y"])
    assert rel_err(ctl["g1til"], g1) > 5 * TOL["bf16"]
