"""Float64 CPU oracle of the GradLev scan (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
``token_weight_scans_b200``) never does, and shares no code with it.

The arithmetic lives in ``gradlev_oracle.cpp`` (serial token-by-token loops
in double / complex<double>, see that file's header for the definition and
its sources); this module builds the shared object with g++ and marshals
numpy arrays through ctypes. The one exception is ``consistency``, which
composes the C++ forward and reverse scans with a few lines of numpy (the
residual, the losses and the consistency term's gradient), written out there.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gradlev_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (-O2, OpenMP, no fast-math). Returns the .so path."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.oracle_fwd_f64.argtypes = [I] * 5 + [P] * 6 + [I]
            lib.oracle_fwd_c128.argtypes = [I] * 5 + [P] * 6 + [I]
            lib.oracle_states_f64.argtypes = [I] * 3 + [P] * 7
            lib.oracle_bwd_f64.argtypes = [I] * 5 + [P] * 11 + [I] * 3
            lib.oracle_fwd_state_f64.argtypes = [I] * 5 + [P] * 8 + [I]
            lib.oracle_fwd_state_c128.argtypes = [I] * 5 + [P] * 8 + [I]
            lib.oracle_bwd_state_f64.argtypes = [I] * 5 + [P] * 14 + [I] * 3
            lib.oracle_serial_f64.argtypes = [I] * 5 + [P] * 7 + [I]
            lib.oracle_serial_c128.argtypes = [I] * 5 + [P] * 7 + [I]
            lib.oracle_decode_f64.argtypes = [I] * 5 + [P] * 8 + [I]
            lib.oracle_mlp2_serial_f64.argtypes = [I] * 6 + [P] * 9 + [I]
            lib.oracle_mlp2_recon_f64.argtypes = [I] * 6 + [P] * 8 + [I] + [P] * 6 + [I]
            lib.oracle_max_threads.restype = I
            _lib = lib
    return _lib


def max_threads() -> int:
    """Threads an oracle call uses when ``nthreads`` is 0 (OpenMP default)."""
    return int(_load().oracle_max_threads())


def _arr(a, dtype):
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dims(x, g):
    B, H, T, din = x.shape
    dout = g.shape[-1]
    assert g.shape == (B, H, T, dout)
    return B, H, T, din, dout


def fwd(x, g, eta, alpha, W0, nthreads: int = 0):
    """y [B,H,T,d_out] of the forward scan. Complex inputs run the complex instantiation."""
    cplx = any(np.iscomplexobj(np.asarray(a)) for a in (x, g, eta, alpha, W0))
    dt = np.complex128 if cplx else np.float64
    x, g, eta, alpha, W0 = (_arr(a, dt) for a in (x, g, eta, alpha, W0))
    B, H, T, din, dout = _dims(x, g)
    assert eta.shape == alpha.shape == (B, H, T) and W0.shape == (H, dout, din)
    y = np.empty((B, H, T, dout), dtype=dt)
    f = _load().oracle_fwd_c128 if cplx else _load().oracle_fwd_f64
    f(B, H, T, din, dout, _p(x), _p(g), _p(eta), _p(alpha), _p(W0), _p(y), int(nthreads))
    return y


def _state_arg(S, dt, B, H, din, dout):
    if S is None:
        return None
    S = _arr(S, dt)
    assert S.shape == (B, H, dout, din), S.shape
    return S


def _pn(a):
    return _p(a) if a is not None else None


def fwd_state(x, g, eta, alpha, W0, S0=None, nthreads: int = 0):
    """Forward scan continuing from the start deviation S0 ([B,H,d_out,d_in], None = 0).

    Returns (y [B,H,T,d_out], S_T [B,H,d_out,d_in]). Complex inputs run the complex
    instantiation."""
    cplx = any(np.iscomplexobj(np.asarray(a)) for a in (x, g, eta, alpha, W0)
               if a is not None) or (S0 is not None and np.iscomplexobj(np.asarray(S0)))
    dt = np.complex128 if cplx else np.float64
    x, g, eta, alpha, W0 = (_arr(a, dt) for a in (x, g, eta, alpha, W0))
    B, H, T, din, dout = _dims(x, g)
    assert eta.shape == alpha.shape == (B, H, T) and W0.shape == (H, dout, din)
    S0 = _state_arg(S0, dt, B, H, din, dout)
    y = np.empty((B, H, T, dout), dtype=dt)
    ST = np.empty((B, H, dout, din), dtype=dt)
    f = _load().oracle_fwd_state_c128 if cplx else _load().oracle_fwd_state_f64
    f(B, H, T, din, dout, _p(x), _p(g), _p(eta), _p(alpha), _p(W0), _pn(S0), _p(y), _p(ST),
      int(nthreads))
    return y, ST


def bwd_state(x, g, eta, alpha, W0, dy, S0=None, LamT=None, ckpt: int = 64,
              mutate: bool = False, nthreads: int = 0):
    """Reverse scan with the carried state: S0 is the start deviation the forward began
    from, LamT the gradient of the objective with respect to S_T (both [B,H,d_out,d_in],
    None = 0). Returns dict dx, dg, deta, dalpha, dW0, dS0."""
    x, g, eta, alpha, W0, dy = (_arr(a, np.float64) for a in (x, g, eta, alpha, W0, dy))
    B, H, T, din, dout = _dims(x, g)
    assert dy.shape == g.shape and W0.shape == (H, dout, din)
    S0 = _state_arg(S0, np.float64, B, H, din, dout)
    LamT = _state_arg(LamT, np.float64, B, H, din, dout)
    out = dict(dx=np.empty_like(x), dg=np.empty_like(g), deta=np.empty_like(eta),
               dalpha=np.empty_like(alpha), dW0=np.empty_like(W0),
               dS0=np.empty((B, H, dout, din)))
    _load().oracle_bwd_state_f64(B, H, T, din, dout, _p(x), _p(g), _p(eta), _p(alpha), _p(W0),
                                 _pn(S0), _p(dy), _pn(LamT), _p(out["dx"]), _p(out["dg"]),
                                 _p(out["deta"]), _p(out["dalpha"]), _p(out["dW0"]),
                                 _p(out["dS0"]), int(ckpt), 1 if mutate else 0, int(nthreads))
    return out


def states(x, g, eta, alpha, W0):
    """(y [T,d_out], S [T+1,d_out,d_in]) for ONE scan given as 2-D/1-D arrays."""
    x, g, eta, alpha, W0 = (_arr(a, np.float64) for a in (x, g, eta, alpha, W0))
    T, din = x.shape
    dout = g.shape[1]
    y = np.empty((T, dout))
    S = np.empty((T + 1, dout, din))
    _load().oracle_states_f64(T, din, dout, _p(x), _p(g), _p(eta), _p(alpha), _p(W0),
                              _p(y), _p(S))
    return y, S


def bwd(x, g, eta, alpha, W0, dy, ckpt: int = 64, mutate: bool = False, nthreads: int = 0):
    """Reverse scan. Returns dict dx, dg, deta, dalpha, dW0 (dW0 summed over b)."""
    x, g, eta, alpha, W0, dy = (_arr(a, np.float64) for a in (x, g, eta, alpha, W0, dy))
    B, H, T, din, dout = _dims(x, g)
    assert dy.shape == g.shape and W0.shape == (H, dout, din)
    out = dict(dx=np.empty_like(x), dg=np.empty_like(g), deta=np.empty_like(eta),
               dalpha=np.empty_like(alpha), dW0=np.empty_like(W0))
    _load().oracle_bwd_f64(B, H, T, din, dout, _p(x), _p(g), _p(eta), _p(alpha), _p(W0),
                           _p(dy), _p(out["dx"]), _p(out["dg"]), _p(out["deta"]),
                           _p(out["dalpha"]), _p(out["dW0"]), int(ckpt), 1 if mutate else 0,
                           int(nthreads))
    return out


def serial(x, v, eta, alpha, W0, nthreads: int = 0):
    """Serial online learner with inner loss 0.5||W x - v||^2: returns (y, g*)."""
    cplx = any(np.iscomplexobj(np.asarray(a)) for a in (x, v, eta, alpha, W0))
    dt = np.complex128 if cplx else np.float64
    x, v, eta, alpha, W0 = (_arr(a, dt) for a in (x, v, eta, alpha, W0))
    B, H, T, din, dout = _dims(x, v)
    y = np.empty((B, H, T, dout), dtype=dt)
    gs = np.empty((B, H, T, dout), dtype=dt)
    f = _load().oracle_serial_c128 if cplx else _load().oracle_serial_f64
    f(B, H, T, din, dout, _p(x), _p(v), _p(eta), _p(alpha), _p(W0), _p(y), _p(gs),
      int(nthreads))
    return y, gs


def decode(x, v, eta, alpha, W0, S, nthreads: int = 0):
    """Deployment decode of T tokens from the carried deviation S ([B,H,d_out,d_in]).

    Returns (y, g, S_after): outputs and costates [B,H,T,d_out], and the deviation after the
    last token. S itself is not modified."""
    x, v, eta, alpha, W0 = (_arr(a, np.float64) for a in (x, v, eta, alpha, W0))
    B, H, T, din, dout = _dims(x, v)
    assert eta.shape == alpha.shape == (B, H, T) and W0.shape == (H, dout, din)
    S = np.array(S, dtype=np.float64, copy=True, order="C")
    assert S.shape == (B, H, dout, din)
    y = np.empty((B, H, T, dout))
    g = np.empty((B, H, T, dout))
    _load().oracle_decode_f64(B, H, T, din, dout, _p(x), _p(v), _p(eta), _p(alpha), _p(W0),
                              _p(S), _p(y), _p(g), int(nthreads))
    return y, g, S


def consistency(x, ghat, eta, alpha, W0, v, lam: float = 1.0, nthreads: int = 0):
    """One GradLev training step of the single adapted layer, given predicted costates.

    Cognaptus, "Parallelize the Training, Keep the Learning Serial", section "The
    predictor is constrained by the learner it is supposed to reproduce":
    - the forward runs on the predicted costates ghat;
    - the costates the proposed trajectory implies are reconstructed by
      backpropagating through the layer. For the synthetic test's inner loss
      0.5 ||y - v||^2 that is gtil_t = y_t - v_t;
    - training combines the token loss with a consistency term that pushes ghat
      toward gtil.

    The term's formula is missing from the page. Read as written, with gtil as the
    target (no gradient through it):
        L = sum_t 0.5 ||gtil_t||^2 + lam ||ghat_t - gtil_t||^2.
    The token loss's output gradient is gtil itself, so its gradients are the reverse
    scan with dy = gtil. The consistency term adds 2 lam (ghat - gtil) to d ghat.

    Returns a dict with:
    - y, gtil, r = ghat - gtil;
    - loss_tok and loss_c, per token [B,H,T];
    - dx, dghat, deta, dalpha, dW0, and dv = -gtil."""
    x, ghat, eta, alpha, W0, v = (_arr(a, np.float64) for a in (x, ghat, eta, alpha, W0, v))
    y = fwd(x, ghat, eta, alpha, W0, nthreads=nthreads)
    gtil = y - v
    r = ghat - gtil
    o = bwd(x, ghat, eta, alpha, W0, gtil, nthreads=nthreads)
    return dict(y=y, gtil=gtil, r=r, loss_tok=0.5 * np.sum(gtil * gtil, axis=-1),
                loss_c=np.sum(r * r, axis=-1), dx=o["dx"], dghat=o["dg"] + 2.0 * lam * r,
                deta=o["deta"], dalpha=o["dalpha"], dW0=o["dW0"], dv=-gtil)


def _mlp2_dims(x, v, W1):
    B, H, T, dx = x.shape
    dy = v.shape[-1]
    dh = W1.shape[1]
    assert v.shape == (B, H, T, dy) and W1.shape == (H, dh, dx)
    return B, H, T, dx, dh, dy


def mlp2_serial(x, v, eta, alpha, W1, W2, nthreads: int = 0):
    """Two-layer adapted MLP, serial test-time backpropagation (tanh hidden layer):
    returns (y [B,H,T,dy], g1 [B,H,T,dh], g2 [B,H,T,dy]) - outputs and true costates."""
    x, v, eta, alpha, W1, W2 = (_arr(a, np.float64) for a in (x, v, eta, alpha, W1, W2))
    B, H, T, dx, dh, dy = _mlp2_dims(x, v, W1)
    assert W2.shape == (H, dy, dh)
    y = np.empty((B, H, T, dy))
    g1 = np.empty((B, H, T, dh))
    g2 = np.empty((B, H, T, dy))
    _load().oracle_mlp2_serial_f64(B, H, T, dx, dh, dy, _p(x), _p(v), _p(eta), _p(alpha),
                                   _p(W1), _p(W2), _p(y), _p(g1), _p(g2), int(nthreads))
    return y, g1, g2


def mlp2_recon(x, g1hat, g2hat, v, eta, alpha, W1, W2, control: bool = False,
               nthreads: int = 0):
    """Parallel reconstruction of the two-layer adapted MLP from given costates. Returns
    dict a, h, y, g2til, g1til, dW1 (dW1 = sum_t g1til_t x_t^T per pair)."""
    x, g1hat, g2hat, v, eta, alpha, W1, W2 = (
        _arr(a, np.float64) for a in (x, g1hat, g2hat, v, eta, alpha, W1, W2))
    B, H, T, dx, dh, dy = _mlp2_dims(x, v, W1)
    out = dict(a=np.empty((B, H, T, dh)), h=np.empty((B, H, T, dh)), y=np.empty((B, H, T, dy)),
               g2til=np.empty((B, H, T, dy)), g1til=np.empty((B, H, T, dh)),
               dW1=np.empty((B, H, dh, dx)))
    _load().oracle_mlp2_recon_f64(B, H, T, dx, dh, dy, _p(x), _p(g1hat), _p(g2hat), _p(v),
                                  _p(eta), _p(alpha), _p(W1), _p(W2), 1 if control else 0,
                                  _p(out["a"]), _p(out["h"]), _p(out["y"]), _p(out["g2til"]),
                                  _p(out["g1til"]), _p(out["dW1"]), int(nthreads))
    return out
