"""Pins of the float64 oracle against facts that do not come from the oracle.

Each test checks the oracle (oracle/gradlev_oracle.cpp) against an
independent statement of what the GradLev scan must compute:

* a hand-worked scalar example (tests/golden/scalar_T3.json);
* the closed form of the state as a discounted sum of earlier rank-one
  updates (Cognaptus, "Parallelize the Training, Keep the Learning Serial",
  section "Once the gradient signals are known, the weight trajectory becomes
  parallelizable"), evaluated by brute force on tiny inputs;
* special cases that reduce to dense matrix products (alpha = 1 is strictly
  causal linear attention, eta = 0 is the static layer, alpha = 0 keeps only
  the previous token, T = 1);
* exact recovery of the serial online learner when the true serial costates
  are supplied (same page, sections "The predictor is constrained by the
  learner it is supposed to reproduce" and "The synthetic test checks the
  mechanism, not model quality"), including the learner's outer gradients
  through the fixed-point adjoint;
* derivative checks of every backward output: exact dot-product tests where
  the output is affine in the argument, central differences where it is
  quadratic (x), complex-step for the polynomial dependence on alpha;
* the negative control of the synthetic-test section: using the persistent
  weight instead of the adapted one in the backward must break the
  gradients while leaving the forward unchanged;
* the carried state of a split sequence (same page, same section: the
  recurrence is affine, so partial results combine). This is pinned by
  - the closed form with the start deviation S_0;
  - running the two parts with S_T -> S_0 and dS_0 -> Lam_T handed across,
    which must equal the whole sequence;
  - derivative checks of every output, dS_0 included, for the objective
    with the <Lam_T, S_T> term;
  - closed-form special cases (static gates; alpha_0 = 0 cuts S_0 off);
* the deployment decode (GradLev abstract: token-by-token forward and backward
  passes at deployment). It is pinned by
  - the serial learner, which reaches the same numbers in a different form;
  - the closed form of one step;
  - token-by-token calls, which must equal one call;
  - exact recovery: the scan given the decode's costates reproduces its
    outputs and end state;
* the consistency step (section "The predictor is constrained by the learner
  it is supposed to reproduce"). It is pinned by
  - the fixed point: with the serial learner's true costates the residual,
    the consistency loss and its gradient vanish;
  - complex-step derivatives of the token loss;
  - the closed form of one token;
* the two-layer adapted MLP of the synthetic test (section "The synthetic
  test checks the mechanism, not model quality"). It is pinned by
  - exact recovery of the serial learner's outputs, hidden costates and
    first-matrix gradient;
  - the control (persistent second matrix in the reconstruction): outputs
    unchanged, costates and gradient far off;
  - the closed form of two tokens;
  - the hidden costate as the complex-step gradient of the token loss.
"""

import json
import os

import numpy as np
import pytest

import oracle
from token_weight_scans_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel(a, b):
    a = np.asarray(a)
    b = np.asarray(b)
    den = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den)


def tiny(B=2, H=2, T=12, d_in=5, d_out=4, seed=7, alpha_mode="sigmoid", with_v=False):
    d = inputs.draw(B, H, T, d_in, d_out, dtype="f32", alpha_mode=alpha_mode, seed=seed,
                    with_v=with_v)
    return {k: v.astype(np.float64) for k, v in d.items()}


# --------------------------------------------------------------------------- golden


def test_golden_scalar_example():
    gd = json.load(open(os.path.join(GOLDEN, "scalar_T3.json")))
    i, e = gd["inputs"], gd["expected"]
    x = np.array(i["x"]).reshape(1, 1, 3, 1)
    g = np.array(i["g"]).reshape(1, 1, 3, 1)
    eta = np.array(i["eta"]).reshape(1, 1, 3)
    alpha = np.array(i["alpha"]).reshape(1, 1, 3)
    W0 = np.array([[[i["W0"]]]])
    dy = np.array(i["dy"]).reshape(1, 1, 3, 1)
    y = oracle.fwd(x, g, eta, alpha, W0)
    assert np.array_equal(y.ravel(), np.array(e["y"]))
    o = oracle.bwd(x, g, eta, alpha, W0, dy, ckpt=2)
    for k in ("dx", "dg", "deta", "dalpha"):
        assert np.array_equal(o[k].ravel(), np.array(e[k])), k
    assert o["dW0"].ravel()[0] == e["dW0"]


# --------------------------------------------------------------------------- closed form


def closed_form(x, g, eta, alpha, W0):
    """S_t = -sum_{s<t} (prod_{r=s+1}^{t-1} alpha_r) eta_s g_s x_s^T, y_t = (W0 + S_t) x_t."""
    T, din = x.shape
    dout = g.shape[1]
    y = np.zeros((T, dout))
    S = np.zeros((T + 1, dout, din))
    for t in range(T + 1):
        acc = np.zeros((dout, din))
        for s in range(t):
            p = 1.0
            for r in range(s + 1, t):
                p *= alpha[r]
            acc -= p * eta[s] * np.outer(g[s], x[s])
        S[t] = acc
        if t < T:
            y[t] = (W0 + acc) @ x[t]
    return y, S


@pytest.mark.parametrize("alpha_mode", ["sigmoid", "log_uniform"])
def test_closed_form_bruteforce(alpha_mode):
    d = tiny(alpha_mode=alpha_mode)
    y = oracle.fwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"])
    B, H = d["x"].shape[:2]
    for b in range(B):
        for h in range(H):
            yc, Sc = closed_form(d["x"][b, h], d["g"][b, h], d["eta"][b, h], d["alpha"][b, h],
                                 d["W0"][h])
            assert rel(y[b, h], yc) < 1e-13
            y1, S1 = oracle.states(d["x"][b, h], d["g"][b, h], d["eta"][b, h],
                                   d["alpha"][b, h], d["W0"][h])
            assert rel(S1, Sc) < 1e-13
            assert rel(y1, yc) < 1e-13


def test_closed_form_random_gates_wide_range():
    # gates spanning [0, 1] including exact zeros and ones
    rng = np.random.default_rng(3)
    T, din, dout = 15, 3, 6
    x = rng.standard_normal((T, din))
    g = rng.standard_normal((T, dout))
    eta = rng.uniform(0, 1, T)
    alpha = rng.choice([0.0, 1.0, 0.3, 0.99], T)
    W0 = rng.standard_normal((dout, din))
    yc, Sc = closed_form(x, g, eta, alpha, W0)
    y1, S1 = oracle.states(x, g, eta, alpha, W0)
    assert rel(y1, yc) < 1e-13 and rel(S1, Sc) < 1e-13


# --------------------------------------------------------------------------- special cases


def test_alpha_one_is_causal_linear_attention():
    d = tiny(T=20)
    d["alpha"][:] = 1.0
    y = oracle.fwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"])
    for b in range(2):
        for h in range(2):
            X, G, e = d["x"][b, h], d["g"][b, h], d["eta"][b, h]
            ref = X @ d["W0"][h].T - np.tril(X @ X.T, -1) @ (e[:, None] * G)
            assert rel(y[b, h], ref) < 1e-13


def test_eta_zero_is_static_layer():
    d = tiny()
    d["eta"][:] = 0.0
    y = oracle.fwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"])
    ref = np.einsum("bhtk,hnk->bhtn", d["x"], d["W0"])
    assert rel(y, ref) < 1e-14


def test_alpha_zero_keeps_previous_token_only():
    d = tiny()
    d["alpha"][:] = 0.0
    y = oracle.fwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"])
    X, G, e = d["x"], d["g"], d["eta"]
    ref = np.einsum("bhtk,hnk->bhtn", X, d["W0"])
    dots = np.einsum("bhtk,bhtk->bht", X[:, :, 1:], X[:, :, :-1])
    ref[:, :, 1:] -= (e[:, :, :-1] * dots)[..., None] * G[:, :, :-1]
    assert rel(y, ref) < 1e-14


def test_single_token():
    d = tiny(T=1)
    y = oracle.fwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"])
    ref = np.einsum("bhtk,hnk->bhtn", d["x"], d["W0"])
    assert np.array_equal(y, ref) or rel(y, ref) < 1e-15
    o = oracle.bwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"], d["dy"])
    assert np.all(o["dg"] == 0) and np.all(o["deta"] == 0) and np.all(o["dalpha"] == 0)
    assert rel(o["dx"], np.einsum("bhtn,hnk->bhtk", d["dy"], d["W0"])) < 1e-14


# --------------------------------------------------------------------------- exact recovery


def test_exact_recovery_of_serial_learner():
    d = tiny(T=40, d_in=6, d_out=5, with_v=True)
    ys, gs = oracle.serial(d["x"], d["v"], d["eta"], d["alpha"], d["W0"])
    y = oracle.fwd(d["x"], gs, d["eta"], d["alpha"], d["W0"])
    assert rel(y, ys) < 1e-12
    # the costates the scan's outputs imply equal the ones that were supplied
    assert rel(y - d["v"], gs) < 1e-12


def _scan_outer_grads(d, gs, u, mutate=False):
    """Outer gradient of L = sum u.y of the serial learner, through the scan and the
    fixed point g = y - v: nu = bwd(u + nu).dg iterated T+1 times (exact, since dg_t
    only depends on upstream at later tokens)."""
    T = d["x"].shape[2]
    nu = np.zeros_like(u)
    for _ in range(T + 1):
        nu = oracle.bwd(d["x"], gs, d["eta"], d["alpha"], d["W0"], u + nu, mutate=mutate)["dg"]
    o = oracle.bwd(d["x"], gs, d["eta"], d["alpha"], d["W0"], u + nu, mutate=mutate)
    return dict(W0=o["dW0"], x=o["dx"], v=-nu, eta=o["deta"], alpha=o["dalpha"])


def _serial_outer_grads(d, u, h=1e-30):
    """Same gradient by complex-step through the serial learner, one entry at a time."""
    out = {}
    for name in ("W0", "x", "v", "eta", "alpha"):
        base = d[name]
        gr = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            args = {k: d[k].astype(np.complex128) for k in ("x", "v", "eta", "alpha", "W0")}
            args[name][idx] += 1j * h
            y, _ = oracle.serial(args["x"], args["v"], args["eta"], args["alpha"], args["W0"])
            gr[idx] = np.sum(y * u).imag / h
        out[name] = gr
    return out


def test_exact_recovery_outer_gradients():
    d = tiny(B=2, H=1, T=7, d_in=3, d_out=2, with_v=True, seed=11)
    u = d["dy"]
    _, gs = oracle.serial(d["x"], d["v"], d["eta"], d["alpha"], d["W0"])
    scan = _scan_outer_grads(d, gs, u)
    ref = _serial_outer_grads(d, u)
    for k in ref:
        assert rel(scan[k], ref[k]) < 1e-12, k


def test_negative_control_persistent_weight_in_backward():
    """Persistent W0^T in place of the adapted weight in the backward: the forward is
    untouched (it does not read the flag) but the gradients are far off."""
    d = tiny(B=2, H=1, T=7, d_in=3, d_out=2, with_v=True, seed=11)
    u = d["dy"]
    _, gs = oracle.serial(d["x"], d["v"], d["eta"], d["alpha"], d["W0"])
    ref = _serial_outer_grads(d, u)
    good = _scan_outer_grads(d, gs, u)
    bad = _scan_outer_grads(d, gs, u, mutate=True)
    assert rel(good["x"], ref["x"]) < 1e-12
    assert rel(bad["x"], ref["x"]) > 1e-3
    # and the plain derivative pin below catches the mutation too
    o_bad = oracle.bwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"], u, mutate=True)
    fd = _fd_grad(d, "x", u)
    assert rel(o_bad["dx"], fd) > 1e-3


# --------------------------------------------------------------------------- derivatives


def _L(d, u, **over):
    a = {k: over.get(k, d[k]) for k in ("x", "g", "eta", "alpha", "W0")}
    y = oracle.fwd(a["x"], a["g"], a["eta"], a["alpha"], a["W0"])
    return np.sum(y * u)


def _fd_grad(d, name, u):
    """Elementwise derivative of L = sum u.y: exact two-point differences for the
    affine arguments (g, eta, W0), central differences for x (L is quadratic in x,
    so they carry no truncation error), complex step for alpha."""
    base = d[name]
    gr = np.zeros_like(base)
    for idx in np.ndindex(base.shape):
        if name == "alpha":
            a = base.astype(np.complex128)
            h = 1e-30
            a[idx] += 1j * h
            gr[idx] = np.imag(_L(d, u, alpha=a)) / h
        elif name == "x":
            h = 1e-3
            p = base.copy(); p[idx] += h
            m = base.copy(); m[idx] -= h
            gr[idx] = (_L(d, u, x=p) - _L(d, u, x=m)) / (2 * h)
        else:
            h = 1.0
            p = base.copy(); p[idx] += h
            gr[idx] = _L(d, u, **{name: p}) - _L(d, u)
    return gr


@pytest.mark.parametrize("alpha_mode", ["sigmoid", "log_uniform"])
def test_backward_matches_derivatives(alpha_mode):
    d = tiny(B=2, H=2, T=9, d_in=5, d_out=4, seed=5, alpha_mode=alpha_mode)
    u = d["dy"]
    o = oracle.bwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"], u, ckpt=4)
    names = dict(x="dx", g="dg", eta="deta", alpha="dalpha", W0="dW0")
    for p, k in names.items():
        fd = _fd_grad(d, p, u)
        tol = 1e-9 if p == "x" else 1e-12
        assert rel(o[k], fd) < tol, (p, rel(o[k], fd))


def test_backward_with_degenerate_gates():
    """alpha in {0, 1} and eta = 0 entries: the derivative is still exact."""
    d = tiny(B=1, H=1, T=10, d_in=3, d_out=4, seed=9)
    d["alpha"][0, 0, ::3] = 0.0
    d["alpha"][0, 0, 1::3] = 1.0
    d["eta"][0, 0, 2] = 0.0
    u = d["dy"]
    o = oracle.bwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"], u, ckpt=3)
    for p, k in dict(x="dx", g="dg", eta="deta", alpha="dalpha", W0="dW0").items():
        fd = _fd_grad(d, p, u)
        assert rel(o[k], fd) < (1e-9 if p == "x" else 1e-12), p


def test_structural_zeros_and_checkpoint_invariance():
    d = tiny(B=2, H=3, T=17, d_in=4, d_out=3, seed=2)
    outs = [oracle.bwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"], d["dy"], ckpt=c)
            for c in (1, 5, 64)]
    o = outs[0]
    assert np.all(o["dg"][:, :, -1] == 0) and np.all(o["deta"][:, :, -1] == 0)
    assert np.all(o["dalpha"][:, :, -1] == 0) and np.all(o["dalpha"][:, :, 0] == 0)
    for other in outs[1:]:
        for k in o:
            assert np.array_equal(o[k], other[k]), k


# --------------------------------------------------------------------------- carried state


def closed_form_state(x, g, eta, alpha, W0, S0):
    """The closed form above plus the carried start deviation:
    S_t = (prod_{r<t} alpha_r) S_0 - sum_{s<t} (prod_{r=s+1}^{t-1} alpha_r) eta_s g_s x_s^T."""
    _, S = closed_form(x, g, eta, alpha, W0)
    T = x.shape[0]
    y = np.zeros((T, g.shape[1]))
    for t in range(T + 1):
        p = 1.0
        for r in range(t):
            p *= alpha[r]
        S[t] = S[t] + p * S0
        if t < T:
            y[t] = (W0 + S[t]) @ x[t]
    return y, S


def _state_inputs(B=1, H=2, T=11, d_in=4, d_out=3, seed=21, alpha_mode="sigmoid"):
    d = tiny(B=B, H=H, T=T, d_in=d_in, d_out=d_out, seed=seed, alpha_mode=alpha_mode)
    rng = np.random.default_rng(seed + 1000)
    S0 = rng.standard_normal((B, H, d_out, d_in))
    LamT = rng.standard_normal((B, H, d_out, d_in))
    return d, S0, LamT


@pytest.mark.parametrize("alpha_mode", ["sigmoid", "log_uniform"])
def test_state_closed_form_bruteforce(alpha_mode):
    d, S0, _ = _state_inputs(B=2, alpha_mode=alpha_mode)
    y, ST = oracle.fwd_state(d["x"], d["g"], d["eta"], d["alpha"], d["W0"], S0)
    B, H = d["x"].shape[:2]
    for b in range(B):
        for h in range(H):
            yc, Sc = closed_form_state(d["x"][b, h], d["g"][b, h], d["eta"][b, h],
                                       d["alpha"][b, h], d["W0"][h], S0[b, h])
            assert rel(y[b, h], yc) < 1e-13
            assert rel(ST[b, h], Sc[-1]) < 1e-13
    # no start state is the zero start state, and matches the stateless forward bit for bit
    y0, _ = oracle.fwd_state(d["x"], d["g"], d["eta"], d["alpha"], d["W0"])
    yz, _ = oracle.fwd_state(d["x"], d["g"], d["eta"], d["alpha"], d["W0"], np.zeros_like(S0))
    assert np.array_equal(y0, oracle.fwd(d["x"], d["g"], d["eta"], d["alpha"], d["W0"]))
    assert np.array_equal(y0, yz)


def _cut(d, t0, t1):
    return {k: (v[:, :, t0:t1] if k != "W0" else v) for k, v in d.items()}


@pytest.mark.parametrize("split", [1, 5, 10])
def test_split_sequence_equals_whole(split):
    d, S0, LamT = _state_inputs(B=2, H=2, T=11)
    T = d["x"].shape[2]
    a, b = _cut(d, 0, split), _cut(d, split, T)
    args = lambda p: (p["x"], p["g"], p["eta"], p["alpha"], p["W0"])
    yw, STw = oracle.fwd_state(*args(d), S0)
    y1, S1 = oracle.fwd_state(*args(a), S0)
    y2, S2 = oracle.fwd_state(*args(b), S1)
    # the same serial arithmetic in the same order: bit for bit
    assert np.array_equal(np.concatenate([y1, y2], axis=2), yw)
    assert np.array_equal(S2, STw)
    w = oracle.bwd_state(*args(d), d["dy"], S0=S0, LamT=LamT, ckpt=3)
    o2 = oracle.bwd_state(*args(b), b["dy"], S0=S1, LamT=LamT, ckpt=3)
    o1 = oracle.bwd_state(*args(a), a["dy"], S0=S0, LamT=o2["dS0"], ckpt=3)
    for k in ("dx", "dg", "deta", "dalpha"):
        assert np.array_equal(np.concatenate([o1[k], o2[k]], axis=2), w[k]), k
    assert np.array_equal(o1["dS0"], w["dS0"])
    assert rel(o1["dW0"] + o2["dW0"], w["dW0"]) < 1e-14


def _L_state(d, u, S0, LamT, over=None):
    over = over or {}
    a = {k: over.get(k, d[k]) for k in ("x", "g", "eta", "alpha", "W0")}
    S0 = over.get("S0", S0)
    y, ST = oracle.fwd_state(a["x"], a["g"], a["eta"], a["alpha"], a["W0"], S0)
    return np.sum(y * u) + np.sum(ST * LamT)


def _fd_grad_state(d, S0, LamT, name, u):
    """Derivatives of L = sum u.y + <Lam_T, S_T>: complex step for alpha, central
    differences for x (quadratic), exact two-point differences for the affine rest."""
    base = S0 if name == "S0" else d[name]
    gr = np.zeros_like(base)
    for idx in np.ndindex(base.shape):
        if name == "alpha":
            a = base.astype(np.complex128)
            h = 1e-30
            a[idx] += 1j * h
            gr[idx] = np.imag(_L_state(d, u, S0, LamT, {"alpha": a})) / h
        elif name == "x":
            h = 1e-3
            p = base.copy(); p[idx] += h
            m = base.copy(); m[idx] -= h
            gr[idx] = (_L_state(d, u, S0, LamT, {"x": p}) - _L_state(d, u, S0, LamT, {"x": m})) / (2 * h)
        else:
            p = base.copy(); p[idx] += 1.0
            gr[idx] = _L_state(d, u, S0, LamT, {name: p}) - _L_state(d, u, S0, LamT)
    return gr


@pytest.mark.parametrize("alpha_mode", ["sigmoid", "log_uniform"])
def test_state_backward_matches_derivatives(alpha_mode):
    d, S0, LamT = _state_inputs(B=1, H=2, T=7, d_in=3, d_out=2, seed=31, alpha_mode=alpha_mode)
    u = d["dy"]
    o = oracle.bwd_state(d["x"], d["g"], d["eta"], d["alpha"], d["W0"], u, S0=S0, LamT=LamT,
                         ckpt=3)
    names = dict(x="dx", g="dg", eta="deta", alpha="dalpha", W0="dW0", S0="dS0")
    for p, k in names.items():
        fd = _fd_grad_state(d, S0, LamT, p, u)
        tol = 1e-9 if p == "x" else 1e-12
        assert rel(o[k], fd) < tol, (p, rel(o[k], fd))


def test_state_special_cases_closed_form():
    d, S0, LamT = _state_inputs(B=1, H=1, T=6, d_in=3, d_out=2, seed=41)
    x, u = d["x"][0, 0], d["dy"][0, 0]
    # static gates (alpha = 1, eta = 0): y_t = (W0 + S0) x_t, S_T = S0,
    # dS0 = Lam_T + sum_t u_t x_t^T
    st = dict(d, alpha=np.ones_like(d["alpha"]), eta=np.zeros_like(d["eta"]))
    y, ST = oracle.fwd_state(st["x"], st["g"], st["eta"], st["alpha"], st["W0"], S0)
    assert rel(y[0, 0], x @ (st["W0"][0] + S0[0, 0]).T) < 1e-14
    assert np.array_equal(ST, S0)
    o = oracle.bwd_state(st["x"], st["g"], st["eta"], st["alpha"], st["W0"], st["dy"], S0=S0,
                         LamT=LamT)
    assert rel(o["dS0"][0, 0], LamT[0, 0] + u.T @ x) < 1e-14
    # alpha_0 = 0 forgets S0 after the first token: only y_0 sees it
    cut = dict(d, alpha=d["alpha"].copy())
    cut["alpha"][0, 0, 0] = 0.0
    y1, ST1 = oracle.fwd_state(cut["x"], cut["g"], cut["eta"], cut["alpha"], cut["W0"], S0)
    y2, ST2 = oracle.fwd_state(cut["x"], cut["g"], cut["eta"], cut["alpha"], cut["W0"])
    assert np.array_equal(y1[:, :, 1:], y2[:, :, 1:]) and np.array_equal(ST1, ST2)
    o = oracle.bwd_state(cut["x"], cut["g"], cut["eta"], cut["alpha"], cut["W0"], cut["dy"],
                         S0=S0, LamT=LamT)
    assert rel(o["dS0"][0, 0], np.outer(u[0], x[0])) < 1e-14


# --------------------------------------------------------------------------- deployment decode


def _decode_inputs(B=2, H=2, T=9, d_in=5, d_out=4, seed=61):
    d = tiny(B=B, H=H, T=T, d_in=d_in, d_out=d_out, seed=seed, with_v=True)
    S0 = np.random.default_rng(seed + 7).standard_normal((B, H, d_out, d_in)) * 0.3
    return d, S0


def test_decode_equals_serial_learner():
    d, _ = _decode_inputs()
    B, H, T, din = d["x"].shape
    zero = np.zeros((B, H, d["v"].shape[-1], din))
    y, g, _ = oracle.decode(d["x"], d["v"], d["eta"], d["alpha"], d["W0"], zero)
    ys, gs = oracle.serial(d["x"], d["v"], d["eta"], d["alpha"], d["W0"])
    assert rel(y, ys) < 1e-14 and rel(g, gs) < 1e-14


def test_decode_single_step_closed_form():
    d, S0 = _decode_inputs(T=1)
    y, g, S1 = oracle.decode(d["x"], d["v"], d["eta"], d["alpha"], d["W0"], S0)
    B, H = S0.shape[:2]
    for b in range(B):
        for h in range(H):
            x, v = d["x"][b, h, 0], d["v"][b, h, 0]
            yc = (d["W0"][h] + S0[b, h]) @ x
            gc = yc - v
            Sc = d["alpha"][b, h, 0] * S0[b, h] - d["eta"][b, h, 0] * np.outer(gc, x)
            assert rel(y[b, h, 0], yc) < 1e-15 and rel(g[b, h, 0], gc) < 1e-14
            assert rel(S1[b, h], Sc) < 1e-15


def test_decode_token_by_token_equals_one_call():
    d, S0 = _decode_inputs(T=7)
    y, g, S = oracle.decode(d["x"], d["v"], d["eta"], d["alpha"], d["W0"], S0)
    St = S0
    for t in range(7):
        sl = lambda a: a[:, :, t:t + 1]
        yt, gt, St = oracle.decode(sl(d["x"]), sl(d["v"]), sl(d["eta"]), sl(d["alpha"]),
                                   d["W0"], St)
        assert np.array_equal(yt, y[:, :, t:t + 1]) and np.array_equal(gt, g[:, :, t:t + 1])
    assert np.array_equal(St, S)


def test_scan_with_decode_costates_recovers_decode():
    """Exact recovery with a carried state: the scan driven by the decode's own costates
    reproduces its outputs and its end deviation."""
    d, S0 = _decode_inputs(T=13)
    y, g, S = oracle.decode(d["x"], d["v"], d["eta"], d["alpha"], d["W0"], S0)
    ys, Ss = oracle.fwd_state(d["x"], g, d["eta"], d["alpha"], d["W0"], S0)
    assert rel(ys, y) < 1e-13 and rel(Ss, S) < 1e-13


# --------------------------------------------------------------------------- consistency step


def test_consistency_vanishes_at_the_serial_costates():
    """Exact consistency: feeding the serial learner's true costates as the prediction
    gives a zero residual, so the consistency term and its gradient vanish."""
    d = tiny(B=2, H=2, T=15, d_in=5, d_out=4, seed=71, with_v=True)
    _, gstar = oracle.serial(d["x"], d["v"], d["eta"], d["alpha"], d["W0"])
    c = oracle.consistency(d["x"], gstar, d["eta"], d["alpha"], d["W0"], d["v"], lam=3.0)
    scale = np.max(np.abs(gstar))
    assert np.max(np.abs(c["r"])) < 1e-14 * scale
    assert np.max(c["loss_c"]) < 1e-27 * scale ** 2
    tok = oracle.bwd(d["x"], gstar, d["eta"], d["alpha"], d["W0"], c["gtil"])["dg"]
    assert np.max(np.abs(c["dghat"] - tok)) < 1e-13 * max(np.max(np.abs(tok)), 1.0)
    # and away from the fixed point the residual is not small
    c2 = oracle.consistency(d["x"], gstar * 0.5, d["eta"], d["alpha"], d["W0"], d["v"])
    assert np.max(np.abs(c2["r"])) > 1e-2 * scale


def _token_loss(d, ghat, over=None):
    over = over or {}
    a = {k: over.get(k, d[k]) for k in ("x", "eta", "alpha", "W0", "v")}
    gh = over.get("ghat", ghat)
    y = oracle.fwd(a["x"], gh, a["eta"], a["alpha"], a["W0"])
    gt = y - a["v"]
    return 0.5 * np.sum(gt * gt)


def test_consistency_token_loss_gradients_complex_step():
    d = tiny(B=1, H=2, T=6, d_in=3, d_out=2, seed=73, with_v=True)
    ghat = np.random.default_rng(74).standard_normal(d["v"].shape)
    lam = 0.7
    c = oracle.consistency(d["x"], ghat, d["eta"], d["alpha"], d["W0"], d["v"], lam=lam)
    names = dict(x="dx", ghat="dghat", eta="deta", alpha="dalpha", W0="dW0", v="dv")
    for p, k in names.items():
        base = ghat if p == "ghat" else d[p]
        gr = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            z = base.astype(np.complex128)
            z[idx] += 1e-30j
            gr[idx] = np.imag(_token_loss(d, ghat, {p: z})) / 1e-30
        got = c[k] - (2.0 * lam * c["r"] if p == "ghat" else 0.0)  # the stop-gradient term
        assert rel(got, gr) < 1e-12, (p, rel(got, gr))


def test_consistency_single_token_closed_form():
    d = tiny(B=1, H=1, T=1, d_in=4, d_out=3, seed=75, with_v=True)
    ghat = np.random.default_rng(76).standard_normal(d["v"].shape)
    c = oracle.consistency(d["x"], ghat, d["eta"], d["alpha"], d["W0"], d["v"], lam=2.0)
    x, v, W0 = d["x"][0, 0, 0], d["v"][0, 0, 0], d["W0"][0]
    gt = W0 @ x - v                      # S_0 = 0: y_0 = W0 x_0
    r = ghat[0, 0, 0] - gt
    assert rel(c["gtil"][0, 0, 0], gt) < 1e-15
    assert abs(c["loss_tok"][0, 0, 0] - 0.5 * gt @ gt) < 1e-14 * (gt @ gt)
    assert abs(c["loss_c"][0, 0, 0] - r @ r) < 1e-14 * (r @ r)
    # one token: dx = W0^T gtil, d ghat = 2 lam r (g only feeds later tokens), dW0 = gtil x^T
    assert rel(c["dx"][0, 0, 0], W0.T @ gt) < 1e-15
    assert rel(c["dghat"][0, 0, 0], 4.0 * r) < 1e-15
    assert rel(c["dW0"][0], np.outer(gt, x)) < 1e-15


# --------------------------------------------------------------------------- two-layer MLP


def _mlp2_inputs(B=1, H=2, T=20, dx=5, dh=4, dy=3, seed=81):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, H, T, dx))
    v = rng.standard_normal((B, H, T, dy))
    eta = rng.uniform(0.0, 0.5, (B, H, T))
    alpha = rng.uniform(0.5, 1.0, (B, H, T))
    W1 = 0.5 * rng.standard_normal((H, dh, dx))
    W2 = 0.5 * rng.standard_normal((H, dy, dh))
    return x, v, eta, alpha, W1, W2


def test_mlp2_exact_recovery_of_serial_learner():
    """The mechanism of the synthetic test: with the serial learner's costates supplied,
    the parallel reconstruction gives its outputs, hidden costates and first-matrix
    gradient back (the pages report rounding-scale differences)."""
    x, v, eta, alpha, W1, W2 = _mlp2_inputs()
    y, g1, g2 = oracle.mlp2_serial(x, v, eta, alpha, W1, W2)
    r = oracle.mlp2_recon(x, g1, g2, v, eta, alpha, W1, W2)
    assert rel(r["y"], y) < 1e-14 and rel(r["g2til"], g2) < 1e-14 and rel(r["g1til"], g1) < 1e-14
    dW1 = np.einsum("bhtk,bhtm->bhkm", g1, x)
    assert rel(r["dW1"], dW1) < 1e-14


def test_mlp2_control_breaks_the_backward_only():
    x, v, eta, alpha, W1, W2 = _mlp2_inputs(seed=83)
    y, g1, g2 = oracle.mlp2_serial(x, v, eta, alpha, W1, W2)
    r = oracle.mlp2_recon(x, g1, g2, v, eta, alpha, W1, W2)
    c = oracle.mlp2_recon(x, g1, g2, v, eta, alpha, W1, W2, control=True)
    assert np.array_equal(c["y"], r["y"]) and np.array_equal(c["g2til"], r["g2til"])
    assert rel(c["g1til"], g1) > 0.05 and rel(c["dW1"], r["dW1"]) > 0.05


def test_mlp2_two_tokens_closed_form():
    x, v, eta, alpha, W1, W2 = _mlp2_inputs(B=1, H=1, T=2, seed=85)
    y, g1, g2 = oracle.mlp2_serial(x, v, eta, alpha, W1, W2)
    X, V, e, al, A, Bm = x[0, 0], v[0, 0], eta[0, 0], alpha[0, 0], W1[0], W2[0]
    # token 0 from the persistent weights
    h0 = np.tanh(A @ X[0]); y0 = Bm @ h0; q0 = y0 - V[0]; p0 = (1 - h0 ** 2) * (Bm.T @ q0)
    # both deviations after token 0
    S1 = -e[0] * np.outer(p0, X[0]); S2 = -e[0] * np.outer(q0, h0)
    h1 = np.tanh((A + S1) @ X[1]); y1 = (Bm + S2) @ h1; q1 = y1 - V[1]
    p1 = (1 - h1 ** 2) * ((Bm + S2).T @ q1)
    assert rel(y[0, 0], np.stack([y0, y1])) < 1e-15
    assert rel(g2[0, 0], np.stack([q0, q1])) < 1e-15
    assert rel(g1[0, 0], np.stack([p0, p1])) < 1e-14


def test_mlp2_hidden_costate_is_the_token_gradient():
    """g1 is the derivative of the token loss with respect to the hidden pre-activation,
    the weights held at their values for that token (complex step on a_0)."""
    x, v, eta, alpha, W1, W2 = _mlp2_inputs(B=1, H=1, T=1, seed=87)
    _, g1, _ = oracle.mlp2_serial(x, v, eta, alpha, W1, W2)
    a0 = W1[0] @ x[0, 0, 0]
    for k in range(a0.size):
        z = a0.astype(np.complex128)
        z[k] += 1e-30j
        r = W2[0] @ np.tanh(z) - v[0, 0, 0]
        assert abs(np.imag(0.5 * np.sum(r * r)) / 1e-30 - g1[0, 0, 0, k]) < 1e-14
