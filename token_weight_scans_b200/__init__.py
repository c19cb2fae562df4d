"""Python binding of libgradlev.so, the B200 GradLev scan library.

Argument marshalling only: every step of the scans runs in the library's CUDA
kernels. PyTorch provides device memory and the stream. The functions carry
the names of the C entry points declared in ``include/gradlev.h``.

If the shared library is missing or cannot be loaded, every call raises
``GradlevError``; there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

__all__ = [
    "GradlevError", "lib", "gradlev_status_string", "gradlev_scan_supported",
    "gradlev_scan_workspace_bytes", "gradlev_scan_ckpt_bytes", "gradlev_scan_fwd",
    "gradlev_scan_bwd", "gradlev_scan_fwd_state", "gradlev_scan_bwd_state",
    "gradlev_decode_step", "gradlev_consistency_workspace_bytes", "gradlev_consistency_step",
    "gradlev_mlp2_workspace_bytes", "gradlev_mlp2_recon", "gradlev_device_status", "gradlev_last_launch_count", "F32", "BF16", "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgradlev.so")
F32 = 0
BF16 = 1

_ENTRY_POINTS = (
    "gradlev_status_string", "gradlev_scan_supported", "gradlev_scan_workspace_bytes",
    "gradlev_scan_ckpt_bytes", "gradlev_scan_fwd", "gradlev_scan_bwd",
    "gradlev_scan_fwd_state", "gradlev_scan_bwd_state", "gradlev_decode_step",
    "gradlev_consistency_workspace_bytes", "gradlev_consistency_step",
    "gradlev_mlp2_workspace_bytes", "gradlev_mlp2_recon", "gradlev_device_status",
    "gradlev_last_launch_count",
)


class GradlevError(RuntimeError):
    """A C entry point returned a non-OK status, or the library is unavailable."""

    def __init__(self, msg, status=None):
        super().__init__(msg)
        self.status = status


_lib = None


def lib():
    """The loaded ctypes library (loads it on first use; raises GradlevError if absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise GradlevError(f"libgradlev.so not built ({LIB_PATH}); run "
                           "`python -m token_weight_scans_b200.build`")
    try:
        L = ctypes.CDLL(LIB_PATH)
    except OSError as e:  # pragma: no cover - depends on the box
        raise GradlevError(f"cannot load {LIB_PATH}: {e}") from e
    I, Z, P = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    L.gradlev_status_string.argtypes = [I]
    L.gradlev_status_string.restype = ctypes.c_char_p
    L.gradlev_scan_supported.argtypes = [I] * 6
    L.gradlev_scan_supported.restype = I
    L.gradlev_scan_workspace_bytes.argtypes = [I] * 7
    L.gradlev_scan_workspace_bytes.restype = Z
    L.gradlev_scan_ckpt_bytes.argtypes = [I] * 6
    L.gradlev_scan_ckpt_bytes.restype = Z
    L.gradlev_scan_fwd.argtypes = [I] * 6 + [P] * 8 + [Z, P]
    L.gradlev_scan_fwd.restype = I
    L.gradlev_scan_bwd.argtypes = [I] * 6 + [P] * 13 + [Z, P]
    L.gradlev_scan_bwd.restype = I
    L.gradlev_scan_fwd_state.argtypes = [I] * 6 + [P] * 10 + [Z, P]
    L.gradlev_scan_fwd_state.restype = I
    L.gradlev_scan_bwd_state.argtypes = [I] * 6 + [P] * 16 + [Z, P]
    L.gradlev_scan_bwd_state.restype = I
    L.gradlev_decode_step.argtypes = [I] * 6 + [P] * 9
    L.gradlev_decode_step.restype = I
    L.gradlev_consistency_workspace_bytes.argtypes = [I] * 6
    L.gradlev_consistency_workspace_bytes.restype = Z
    L.gradlev_consistency_step.argtypes = ([I] * 6 + [P] * 6 + [ctypes.c_float] + [P] * 11 +
                                           [Z, P])
    L.gradlev_consistency_step.restype = I
    L.gradlev_mlp2_workspace_bytes.argtypes = [I] * 7
    L.gradlev_mlp2_workspace_bytes.restype = Z
    L.gradlev_mlp2_recon.argtypes = [I] * 7 + [P] * 8 + [I] + [P] * 7 + [Z, P]
    L.gradlev_mlp2_recon.restype = I
    L.gradlev_device_status.argtypes = [P, P]
    L.gradlev_device_status.restype = I
    L.gradlev_last_launch_count.argtypes = []
    L.gradlev_last_launch_count.restype = I
    L.gradlev_debug_inject_timeout.argtypes = [I, I]
    L.gradlev_debug_inject_timeout.restype = None
    L.gradlev_debug_summary_rescale.argtypes = [ctypes.c_float]
    L.gradlev_debug_summary_rescale.restype = None
    _lib = L
    return L


def gradlev_status_string(status: int) -> str:
    return lib().gradlev_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != 0:
        raise GradlevError(f"{what}: {gradlev_status_string(status)}", status)


def _dt_code(dtype) -> int:
    import torch
    if dtype == torch.float32:
        return F32
    if dtype == torch.bfloat16:
        return BF16
    raise GradlevError(f"unsupported I/O dtype {dtype}")


def gradlev_scan_supported(B, H, T, d_in, d_out, dt) -> int:
    return int(lib().gradlev_scan_supported(B, H, T, d_in, d_out, dt))


def gradlev_scan_workspace_bytes(B, H, T, d_in, d_out, dt, is_bwd) -> int:
    return int(lib().gradlev_scan_workspace_bytes(B, H, T, d_in, d_out, dt, int(is_bwd)))


def gradlev_scan_ckpt_bytes(B, H, T, d_in, d_out, dt) -> int:
    return int(lib().gradlev_scan_ckpt_bytes(B, H, T, d_in, d_out, dt))


def gradlev_last_launch_count() -> int:
    return int(lib().gradlev_last_launch_count())


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream_ptr(stream, device=None):
    """The stream as a cudaStream_t: the given one, which must belong to `device`, or the
    current stream of `device` (of the current device when `device` is None)."""
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    if device is not None and stream.device != device:
        raise GradlevError(f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _cuda_device(x):
    """The device of x, which must be a CUDA device: the library's kernels dereference
    every pointer on the GPU, so host memory is refused here, before any call."""
    if not getattr(x, "is_cuda", False):
        raise GradlevError(f"tensors must be on a CUDA device, got {getattr(x, 'device', type(x))}")
    return x.device


def _check_tensor(name, t, shape, dtype, device):
    if t.shape != tuple(shape):
        raise GradlevError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")
    if t.dtype != dtype:
        raise GradlevError(f"{name}: dtype {t.dtype} != {dtype}")
    if t.device != device:
        raise GradlevError(f"{name}: device {t.device} != {device}")
    if not t.is_contiguous():
        raise GradlevError(f"{name}: must be contiguous")


def _check_buffer(name, t, nbytes, device):
    """A caller's byte buffer (workspace, checkpoints): on the call's device, contiguous,
    at least nbytes long."""
    if t.device != device:
        raise GradlevError(f"{name}: device {t.device} != {device}")
    if not t.is_contiguous():
        raise GradlevError(f"{name}: must be contiguous")
    if t.numel() * t.element_size() < nbytes:
        raise GradlevError(f"{name} too small: {t.numel() * t.element_size()} < {nbytes} bytes")


def _workspace(nbytes, device, workspace):
    import torch
    if workspace is None:
        return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    _check_buffer("workspace", workspace, nbytes, device)
    return workspace


def _check_ckpt(ckpt, B, H, T, d_in, d_out, code, device):
    if ckpt is not None:
        _check_buffer("ckpt", ckpt, gradlev_scan_ckpt_bytes(B, H, T, d_in, d_out, code), device)


def _check_out(out, spec, device):
    """Caller-supplied outputs: every tensor of `spec` (name -> (shape, dtype)) present and
    matching; None entries allowed only where spec says so (dtype None)."""
    for k, (shape, dtype) in spec.items():
        t = out.get(k)
        if t is None:
            if dtype is None:
                continue
            raise GradlevError(f"out[{k!r}] missing")
        _check_tensor(f"out[{k!r}]", t, shape, t.dtype if dtype is None else dtype, device)


def _dims(x, g):
    if x.dim() != 4 or g.dim() != 4:
        raise GradlevError("x and g must be [B,H,T,d] tensors")
    B, H, T, d_in = x.shape
    d_out = g.shape[-1]
    return B, H, T, d_in, d_out


def gradlev_scan_fwd(x, g, eta, alpha, W0, *, y=None, ckpt=None, workspace=None, stream=None):
    """Forward scan on the GPU. Returns y [B,H,T,d_out] (dtype of x)."""
    import torch
    B, H, T, d_in, d_out = _dims(x, g)
    dev, dt = _cuda_device(x), x.dtype
    f32 = torch.float32
    _check_tensor("g", g, (B, H, T, d_out), dt, dev)
    _check_tensor("eta", eta, (B, H, T), f32, dev)
    _check_tensor("alpha", alpha, (B, H, T), f32, dev)
    _check_tensor("W0", W0, (H, d_out, d_in), f32, dev)
    _check_tensor("x", x, (B, H, T, d_in), dt, dev)
    code = _dt_code(dt)
    _check(gradlev_scan_supported(B, H, T, d_in, d_out, code), "gradlev_scan_fwd")
    if y is None:
        y = torch.empty((B, H, T, d_out), dtype=dt, device=dev)
    _check_tensor("y", y, (B, H, T, d_out), dt, dev)
    _check_ckpt(ckpt, B, H, T, d_in, d_out, code, dev)
    nws = gradlev_scan_workspace_bytes(B, H, T, d_in, d_out, code, 0)
    ws = _workspace(nws, dev, workspace)
    with torch.cuda.device(dev):  # launches go to the tensors' device
        st = lib().gradlev_scan_fwd(B, H, T, d_in, d_out, code, _ptr(x), _ptr(g), _ptr(eta),
                                    _ptr(alpha), _ptr(W0), _ptr(y), _ptr(ckpt), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream_ptr(stream, dev))
    _check(st, "gradlev_scan_fwd")
    return y


def gradlev_scan_bwd(x, g, eta, alpha, W0, dy, *, ckpt=None, workspace=None, stream=None,
                     out=None):
    """Reverse scan on the GPU. Returns dict dx, dg, deta, dalpha, dW0."""
    import torch
    B, H, T, d_in, d_out = _dims(x, g)
    dev, dt = _cuda_device(x), x.dtype
    f32 = torch.float32
    _check_tensor("x", x, (B, H, T, d_in), dt, dev)
    _check_tensor("g", g, (B, H, T, d_out), dt, dev)
    _check_tensor("dy", dy, (B, H, T, d_out), dt, dev)
    _check_tensor("eta", eta, (B, H, T), f32, dev)
    _check_tensor("alpha", alpha, (B, H, T), f32, dev)
    _check_tensor("W0", W0, (H, d_out, d_in), f32, dev)
    code = _dt_code(dt)
    _check(gradlev_scan_supported(B, H, T, d_in, d_out, code), "gradlev_scan_bwd")
    if out is None:
        out = dict(dx=torch.empty_like(x), dg=torch.empty_like(g),
                   deta=torch.empty((B, H, T), dtype=f32, device=dev),
                   dalpha=torch.empty((B, H, T), dtype=f32, device=dev),
                   dW0=torch.empty((H, d_out, d_in), dtype=f32, device=dev))
    _check_out(out, dict(dx=((B, H, T, d_in), dt), dg=((B, H, T, d_out), dt),
                         deta=((B, H, T), f32), dalpha=((B, H, T), f32),
                         dW0=((H, d_out, d_in), f32)), dev)
    _check_ckpt(ckpt, B, H, T, d_in, d_out, code, dev)
    nws = gradlev_scan_workspace_bytes(B, H, T, d_in, d_out, code, 1)
    ws = _workspace(nws, dev, workspace)
    with torch.cuda.device(dev):  # launches go to the tensors' device
        st = lib().gradlev_scan_bwd(B, H, T, d_in, d_out, code, _ptr(x), _ptr(g), _ptr(eta),
                                    _ptr(alpha), _ptr(W0), _ptr(dy), _ptr(out["dx"]),
                                    _ptr(out["dg"]), _ptr(out["deta"]), _ptr(out["dalpha"]),
                                    _ptr(out["dW0"]), _ptr(ckpt), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream_ptr(stream, dev))
    _check(st, "gradlev_scan_bwd")
    return out


def _state_tensor(name, t, B, H, d_in, d_out, dev):
    import torch
    if t is not None:
        _check_tensor(name, t, (B, H, d_out, d_in), torch.float32, dev)
    return t


def gradlev_scan_fwd_state(x, g, eta, alpha, W0, S0=None, *, y=None, ST=None, ckpt=None,
                           workspace=None, stream=None):
    """Forward scan continuing from the carried deviation S0 ([B,H,d_out,d_in] float32,
    None = 0). Returns (y, ST), ST the deviation after the last token."""
    import torch
    B, H, T, d_in, d_out = _dims(x, g)
    dev, dt = _cuda_device(x), x.dtype
    f32 = torch.float32
    _check_tensor("x", x, (B, H, T, d_in), dt, dev)
    _check_tensor("g", g, (B, H, T, d_out), dt, dev)
    _check_tensor("eta", eta, (B, H, T), f32, dev)
    _check_tensor("alpha", alpha, (B, H, T), f32, dev)
    _check_tensor("W0", W0, (H, d_out, d_in), f32, dev)
    _state_tensor("S0", S0, B, H, d_in, d_out, dev)
    code = _dt_code(dt)
    _check(gradlev_scan_supported(B, H, T, d_in, d_out, code), "gradlev_scan_fwd_state")
    if y is None:
        y = torch.empty((B, H, T, d_out), dtype=dt, device=dev)
    _check_tensor("y", y, (B, H, T, d_out), dt, dev)
    if ST is None:
        ST = torch.empty((B, H, d_out, d_in), dtype=f32, device=dev)
    _state_tensor("ST", ST, B, H, d_in, d_out, dev)
    _check_ckpt(ckpt, B, H, T, d_in, d_out, code, dev)
    nws = gradlev_scan_workspace_bytes(B, H, T, d_in, d_out, code, 0)
    ws = _workspace(nws, dev, workspace)
    with torch.cuda.device(dev):  # launches go to the tensors' device
        st = lib().gradlev_scan_fwd_state(B, H, T, d_in, d_out, code, _ptr(x), _ptr(g), _ptr(eta),
                                          _ptr(alpha), _ptr(W0), _ptr(S0), _ptr(y), _ptr(ST),
                                          _ptr(ckpt), _ptr(ws), ws.numel() * ws.element_size(),
                                          _stream_ptr(stream, dev))
    _check(st, "gradlev_scan_fwd_state")
    return y, ST


def gradlev_scan_bwd_state(x, g, eta, alpha, W0, dy, S0=None, LamT=None, *, ckpt=None,
                           workspace=None, stream=None, out=None):
    """Reverse scan with the carried state: S0 the start deviation of the forward (read only
    without ckpt), LamT the adjoint flowing in after the last token (both [B,H,d_out,d_in]
    float32, None = 0). Returns dict dx, dg, deta, dalpha, dW0, dS0."""
    import torch
    B, H, T, d_in, d_out = _dims(x, g)
    dev, dt = _cuda_device(x), x.dtype
    f32 = torch.float32
    _check_tensor("x", x, (B, H, T, d_in), dt, dev)
    _check_tensor("g", g, (B, H, T, d_out), dt, dev)
    _check_tensor("dy", dy, (B, H, T, d_out), dt, dev)
    _check_tensor("eta", eta, (B, H, T), f32, dev)
    _check_tensor("alpha", alpha, (B, H, T), f32, dev)
    _check_tensor("W0", W0, (H, d_out, d_in), f32, dev)
    _state_tensor("S0", S0, B, H, d_in, d_out, dev)
    _state_tensor("LamT", LamT, B, H, d_in, d_out, dev)
    code = _dt_code(dt)
    _check(gradlev_scan_supported(B, H, T, d_in, d_out, code), "gradlev_scan_bwd_state")
    if out is None:
        out = dict(dx=torch.empty_like(x), dg=torch.empty_like(g),
                   deta=torch.empty((B, H, T), dtype=f32, device=dev),
                   dalpha=torch.empty((B, H, T), dtype=f32, device=dev),
                   dW0=torch.empty((H, d_out, d_in), dtype=f32, device=dev),
                   dS0=torch.empty((B, H, d_out, d_in), dtype=f32, device=dev))
    _check_out(out, dict(dx=((B, H, T, d_in), dt), dg=((B, H, T, d_out), dt),
                         deta=((B, H, T), f32), dalpha=((B, H, T), f32),
                         dW0=((H, d_out, d_in), f32), dS0=((B, H, d_out, d_in), f32)), dev)
    _check_ckpt(ckpt, B, H, T, d_in, d_out, code, dev)
    nws = gradlev_scan_workspace_bytes(B, H, T, d_in, d_out, code, 1)
    ws = _workspace(nws, dev, workspace)
    with torch.cuda.device(dev):  # launches go to the tensors' device
        st = lib().gradlev_scan_bwd_state(B, H, T, d_in, d_out, code, _ptr(x), _ptr(g), _ptr(eta),
                                          _ptr(alpha), _ptr(W0), _ptr(S0), _ptr(dy), _ptr(LamT),
                                          _ptr(out["dx"]), _ptr(out["dg"]), _ptr(out["deta"]),
                                          _ptr(out["dalpha"]), _ptr(out["dW0"]), _ptr(out["dS0"]),
                                          _ptr(ckpt), _ptr(ws), ws.numel() * ws.element_size(),
                                          _stream_ptr(stream, dev))
    _check(st, "gradlev_scan_bwd_state")
    return out


def gradlev_decode_step(x, v, eta, alpha, W0, S, *, y=None, g=None, want_g=True, stream=None):
    """Deployment decode of the T tokens of x in order, from the carried deviation S
    ([B,H,d_out,d_in] float32, updated in place). Returns (y, g): outputs and costates
    [B,H,T,d_out] (g is None when want_g is False and no buffer is given)."""
    import torch
    B, H, T, d_in, d_out = _dims(x, v)
    dev, dt = _cuda_device(x), x.dtype
    f32 = torch.float32
    _check_tensor("x", x, (B, H, T, d_in), dt, dev)
    _check_tensor("v", v, (B, H, T, d_out), dt, dev)
    _check_tensor("eta", eta, (B, H, T), f32, dev)
    _check_tensor("alpha", alpha, (B, H, T), f32, dev)
    _check_tensor("W0", W0, (H, d_out, d_in), f32, dev)
    _check_tensor("S", S, (B, H, d_out, d_in), f32, dev)
    if y is None:
        y = torch.empty((B, H, T, d_out), dtype=dt, device=dev)
    _check_tensor("y", y, (B, H, T, d_out), dt, dev)
    if g is None and want_g:
        g = torch.empty((B, H, T, d_out), dtype=dt, device=dev)
    if g is not None:
        _check_tensor("g", g, (B, H, T, d_out), dt, dev)
    with torch.cuda.device(dev):  # launches go to the tensors' device
        st = lib().gradlev_decode_step(B, H, T, d_in, d_out, _dt_code(dt), _ptr(x), _ptr(v),
                                       _ptr(eta), _ptr(alpha), _ptr(W0), _ptr(S), _ptr(y), _ptr(g),
                                       _stream_ptr(stream, dev))
    _check(st, "gradlev_decode_step")
    return y, g


def gradlev_consistency_workspace_bytes(B, H, T, d_in, d_out, dt) -> int:
    return int(lib().gradlev_consistency_workspace_bytes(B, H, T, d_in, d_out, dt))


def gradlev_consistency_step(x, ghat, eta, alpha, W0, v, lam=1.0, *, want_dv=True,
                             workspace=None, stream=None, out=None):
    """One training step of the adapted layer from predicted costates ghat (see
    include/gradlev.h). Returns dict y, gtil, loss_tok, loss_c, dx, dghat, deta, dalpha, dW0
    and dv (None when want_dv is False)."""
    import torch
    B, H, T, d_in, d_out = _dims(x, ghat)
    dev, dt = _cuda_device(x), x.dtype
    f32 = torch.float32
    _check_tensor("x", x, (B, H, T, d_in), dt, dev)
    _check_tensor("ghat", ghat, (B, H, T, d_out), dt, dev)
    _check_tensor("v", v, (B, H, T, d_out), dt, dev)
    _check_tensor("eta", eta, (B, H, T), f32, dev)
    _check_tensor("alpha", alpha, (B, H, T), f32, dev)
    _check_tensor("W0", W0, (H, d_out, d_in), f32, dev)
    code = _dt_code(dt)
    nws = gradlev_consistency_workspace_bytes(B, H, T, d_in, d_out, code)
    if nws == 0:
        raise GradlevError("gradlev_consistency_step: unsupported shape", 2)
    if out is None:
        out = dict(y=torch.empty_like(ghat), gtil=torch.empty_like(ghat),
                   loss_tok=torch.empty((B, H, T), dtype=f32, device=dev),
                   loss_c=torch.empty((B, H, T), dtype=f32, device=dev),
                   dx=torch.empty_like(x), dghat=torch.empty_like(ghat),
                   deta=torch.empty((B, H, T), dtype=f32, device=dev),
                   dalpha=torch.empty((B, H, T), dtype=f32, device=dev),
                   dW0=torch.empty((H, d_out, d_in), dtype=f32, device=dev),
                   dv=torch.empty_like(ghat) if want_dv else None)
    _check_out(out, dict(y=((B, H, T, d_out), dt), gtil=((B, H, T, d_out), dt),
                         loss_tok=((B, H, T), f32), loss_c=((B, H, T), f32),
                         dx=((B, H, T, d_in), dt), dghat=((B, H, T, d_out), dt),
                         deta=((B, H, T), f32), dalpha=((B, H, T), f32),
                         dW0=((H, d_out, d_in), f32)), dev)
    if out.get("dv") is not None:
        _check_tensor("out['dv']", out["dv"], (B, H, T, d_out), dt, dev)
    ws = _workspace(nws, dev, workspace)
    with torch.cuda.device(dev):  # launches go to the tensors' device
        st = lib().gradlev_consistency_step(
            B, H, T, d_in, d_out, code, _ptr(x), _ptr(ghat), _ptr(eta), _ptr(alpha), _ptr(W0),
            _ptr(v), float(lam), _ptr(out["y"]), _ptr(out["gtil"]), _ptr(out["loss_tok"]),
            _ptr(out["loss_c"]), _ptr(out["dx"]), _ptr(out["dghat"]), _ptr(out["deta"]),
            _ptr(out["dalpha"]), _ptr(out["dW0"]), _ptr(out.get("dv")), _ptr(ws),
            ws.numel() * ws.element_size(), _stream_ptr(stream, dev))
    _check(st, "gradlev_consistency_step")
    return out


def gradlev_mlp2_workspace_bytes(B, H, T, d_x, d_h, d_y, dt) -> int:
    return int(lib().gradlev_mlp2_workspace_bytes(B, H, T, d_x, d_h, d_y, dt))


def gradlev_mlp2_recon(x, g1hat, g2hat, v, eta, alpha, W1, W2, control=False, *,
                       workspace=None, stream=None, out=None):
    """Parallel reconstruction of the two-layer adapted MLP from given costates (see
    include/gradlev.h). Returns dict a, h, y, g2til, g1til, dW1."""
    import torch
    if x.dim() != 4 or v.dim() != 4 or W1.dim() != 3:
        raise GradlevError("x, v must be [B,H,T,d] and W1 [H,d_h,d_x]")
    B, H, T, d_x = x.shape
    d_y = v.shape[-1]
    d_h = W1.shape[1]
    dev, dt = _cuda_device(x), x.dtype
    f32 = torch.float32
    _check_tensor("x", x, (B, H, T, d_x), dt, dev)
    _check_tensor("g1hat", g1hat, (B, H, T, d_h), dt, dev)
    _check_tensor("g2hat", g2hat, (B, H, T, d_y), dt, dev)
    _check_tensor("v", v, (B, H, T, d_y), dt, dev)
    _check_tensor("eta", eta, (B, H, T), f32, dev)
    _check_tensor("alpha", alpha, (B, H, T), f32, dev)
    _check_tensor("W1", W1, (H, d_h, d_x), f32, dev)
    _check_tensor("W2", W2, (H, d_y, d_h), f32, dev)
    code = _dt_code(dt)
    nws = gradlev_mlp2_workspace_bytes(B, H, T, d_x, d_h, d_y, code)
    if nws == 0:
        raise GradlevError("gradlev_mlp2_recon: unsupported shape", 2)
    if out is None:
        out = dict(a=torch.empty_like(g1hat), h=torch.empty_like(g1hat), y=torch.empty_like(v),
                   g2til=torch.empty_like(v), g1til=torch.empty_like(g1hat),
                   dW1=torch.empty((B, H, d_h, d_x), dtype=f32, device=dev))
    _check_out(out, dict(a=((B, H, T, d_h), dt), h=((B, H, T, d_h), dt),
                         y=((B, H, T, d_y), dt), g2til=((B, H, T, d_y), dt),
                         g1til=((B, H, T, d_h), dt), dW1=((B, H, d_h, d_x), f32)), dev)
    ws = _workspace(nws, dev, workspace)
    with torch.cuda.device(dev):  # launches go to the tensors' device
        st = lib().gradlev_mlp2_recon(
            B, H, T, d_x, d_h, d_y, code, _ptr(x), _ptr(g1hat), _ptr(g2hat), _ptr(v), _ptr(eta),
            _ptr(alpha), _ptr(W1), _ptr(W2), 1 if control else 0, _ptr(out["a"]), _ptr(out["h"]),
            _ptr(out["y"]), _ptr(out["g2til"]), _ptr(out["g1til"]), _ptr(out["dW1"]), _ptr(ws),
            ws.numel() * ws.element_size(), _stream_ptr(stream, dev))
    _check(st, "gradlev_mlp2_recon")
    return out


def gradlev_device_status(workspace, stream=None) -> int:
    import torch
    with torch.cuda.device(workspace.device):
        return int(lib().gradlev_device_status(_ptr(workspace),
                                               _stream_ptr(stream, workspace.device)))
