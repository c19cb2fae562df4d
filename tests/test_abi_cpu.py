"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
entry point include/gradlev.h declares, and rejects bad arguments before any launch."""

import ctypes
import os
import re

import pytest

import token_weight_scans_b200 as tw
from token_weight_scans_b200 import build as tw_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gradlev.h")


@pytest.fixture(scope="module")
def L():
    tw_build.build()
    return tw.lib()


def declared_entry_points():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"GRADLEV_API\s+[\w\s\*]+?\b(gradlev_\w+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_entry_points()
    for n in ("gradlev_scan_fwd", "gradlev_scan_bwd", "gradlev_scan_workspace_bytes",
              "gradlev_status_string", "gradlev_scan_supported", "gradlev_scan_ckpt_bytes",
              "gradlev_device_status", "gradlev_last_launch_count", "gradlev_scan_fwd_state",
              "gradlev_scan_bwd_state", "gradlev_decode_step", "gradlev_consistency_step",
              "gradlev_consistency_workspace_bytes", "gradlev_mlp2_recon",
              "gradlev_mlp2_workspace_bytes"):
        assert n in names, n


def test_library_exports_every_declared_symbol(L):
    for n in declared_entry_points():
        assert hasattr(L, n), n


def test_status_strings(L):
    assert tw.gradlev_status_string(0) == "GRADLEV_OK"
    assert tw.gradlev_status_string(3) == "GRADLEV_ERR_WORKSPACE"
    assert tw.gradlev_status_string(99) == "GRADLEV_UNKNOWN_STATUS"


@pytest.mark.parametrize("shape,dt,ok", [
    ((1, 1, 256, 16, 16), 0, 0),
    ((4, 8, 2048, 64, 64), 0, 0),
    ((8, 16, 4096, 128, 128), 1, 0),
    ((1, 1, 1, 8, 8), 1, 0),
    ((0, 1, 4, 16, 16), 0, 1),
    ((1, 1, 4, 16, 16), 7, 1),
    ((1, 1, 4, 6, 16), 0, 2),
    ((1, 1, 4, 16, 12), 0, 2),
    ((1, 1, 4, 256, 256), 0, 2),
    ((1, 16, 32768, 128, 256), 1, 0),
    ((1, 16, 32768, 128, 256), 0, 2),
    ((1, 1, 4, 128, 384), 1, 2),
])
def test_supported_shapes(L, shape, dt, ok):
    assert tw.gradlev_scan_supported(*shape, dt) == ok
    ws = tw.gradlev_scan_workspace_bytes(*shape, dt, 1)
    assert (ws >= 256) == (ok == 0)


def test_bwd_workspace_covers_partials_and_states(L):
    B, H, T, di, do = 2, 3, 100, 16, 24
    ws_f = tw.gradlev_scan_workspace_bytes(B, H, T, di, do, 0, 0)
    ws_b = tw.gradlev_scan_workspace_bytes(B, H, T, di, do, 0, 1)
    ck = tw.gradlev_scan_ckpt_bytes(B, H, T, di, do, 0)
    assert ws_f >= 256
    assert ws_b >= 256 + B * H * di * do * 4 + ck
    assert ck >= B * H * di * do * 4


def test_argument_errors_return_before_launch(L):
    P = ctypes.c_void_p
    fake = P(4096)  # never dereferenced: validation fails first
    # null input
    st = L.gradlev_scan_fwd(1, 1, 8, 16, 16, 0, P(0), fake, fake, fake, fake, fake, P(0), fake,
                            1 << 20, P(0))
    assert st == 1
    # unsupported shape
    st = L.gradlev_scan_fwd(1, 1, 8, 16, 12, 0, fake, fake, fake, fake, fake, fake, P(0), fake,
                            1 << 20, P(0))
    assert st == 2
    # workspace too small
    st = L.gradlev_scan_fwd(1, 1, 8, 16, 16, 0, fake, fake, fake, fake, fake, fake, P(0), fake,
                            16, P(0))
    assert st == 3
    st = L.gradlev_scan_bwd(1, 1, 8, 16, 16, 0, fake, fake, fake, fake, fake, fake, fake, fake,
                            fake, fake, fake, P(0), fake, 16, P(0))
    assert st == 3
    # misaligned pointer
    st = L.gradlev_scan_bwd(1, 1, 8, 16, 16, 0, P(4098), fake, fake, fake, fake, fake, fake,
                            fake, fake, fake, fake, P(0), fake, 1 << 30, P(0))
    assert st == 1
    assert L.gradlev_device_status(P(0), P(0)) == 1


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(tw, "_lib", None)
    monkeypatch.setattr(tw, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(tw.GradlevError):
        tw.lib()


def test_forward_workspace_grows_only_for_segmented_scans(L):
    """Scans that fill the GPU run unsegmented and need only the status word;
    few long scans are cut into segments, whose summaries live in the workspace."""
    full = tw.gradlev_scan_workspace_bytes(8, 16, 4096, 128, 128, tw.BF16, 0)
    few = tw.gradlev_scan_workspace_bytes(1, 2, 4096, 128, 128, tw.BF16, 0)
    assert full == 256
    # 2 scans -> segments; two fp32 [scan][seg][d_out][d_in] buffers at least
    assert few >= 256 + 2 * 2 * 2 * 128 * 128 * 4
    # the reverse scan's workspace covers its per-segment dW0 partials as well
    bwd_few = tw.gradlev_scan_workspace_bytes(1, 2, 4096, 128, 128, tw.BF16, 1)
    bwd_full = tw.gradlev_scan_workspace_bytes(8, 16, 4096, 128, 128, tw.BF16, 1)
    assert bwd_few > tw.gradlev_scan_ckpt_bytes(1, 2, 4096, 128, 128, tw.BF16) + 2 * 128 * 128 * 4
    assert bwd_full >= 256 + 8 * 16 * 128 * 128 * 4 + \
        tw.gradlev_scan_ckpt_bytes(8, 16, 4096, 128, 128, tw.BF16)
    # one chunk: nothing to split
    assert tw.gradlev_scan_workspace_bytes(1, 1, 64, 128, 128, tw.BF16, 0) == 256


def test_state_entry_points_validate_before_launch(L):
    """The carried-state calls check their extra pointers on the host, like the rest."""
    P = ctypes.c_void_p
    fake = P(4096)  # never dereferenced: validation fails first
    I = ctypes.c_int
    L.gradlev_scan_fwd_state.restype = I
    L.gradlev_scan_bwd_state.restype = I
    fwd = lambda S0, ST, ws=1 << 20, d_out=16: L.gradlev_scan_fwd_state(
        1, 1, 8, 16, d_out, 0, fake, fake, fake, fake, fake, S0, fake, ST, P(0), fake, ws, P(0))
    bwd = lambda S0, LamT, dS0, ws=1 << 30: L.gradlev_scan_bwd_state(
        1, 1, 8, 16, 16, 0, fake, fake, fake, fake, fake, S0, fake, LamT, fake, fake, fake, fake,
        fake, dS0, P(0), fake, ws, P(0))
    assert fwd(P(4100), P(0)) == 1  # misaligned S0
    assert fwd(P(0), P(4104)) == 1  # misaligned ST
    assert fwd(P(0), P(0), d_out=12) == 2  # unsupported shape
    assert fwd(P(0), P(0), ws=16) == 3  # workspace too small
    assert bwd(P(4100), P(0), P(0)) == 1
    assert bwd(P(0), P(4100), P(0)) == 1
    assert bwd(P(0), P(0), P(4100)) == 1
    assert bwd(P(0), P(0), P(0), ws=16) == 3
    # the required pointers are still required
    assert L.gradlev_scan_fwd_state(1, 1, 8, 16, 16, 0, P(0), fake, fake, fake, fake, P(0), fake,
                                    P(0), P(0), fake, 1 << 20, P(0)) == 1


def test_decode_step_validates_before_launch(L):
    P = ctypes.c_void_p
    fake = P(4096)
    L.gradlev_decode_step.restype = ctypes.c_int
    call = lambda d_in=16, d_out=8, x=fake, S=fake, T=1: L.gradlev_decode_step(
        1, 1, T, d_in, d_out, 1, x, fake, fake, fake, fake, S, fake, P(0), P(0))
    assert call(d_in=18) == 2            # d_in not a multiple of 4
    assert call(d_in=260) == 2           # d_in above 256
    assert call(T=0) == 1                # empty
    assert call(x=P(0)) == 1             # missing input
    assert call(x=P(4098)) == 1          # bf16 x not aligned to 4 elements
    assert call(S=P(4104)) == 1          # S not 16-byte aligned


def test_consistency_step_validates_before_launch(L):
    P = ctypes.c_void_p
    fake = P(4096)
    I, Z = ctypes.c_int, ctypes.c_size_t
    L.gradlev_consistency_workspace_bytes.restype = Z
    L.gradlev_consistency_workspace_bytes.argtypes = [I] * 6
    L.gradlev_consistency_step.restype = I
    L.gradlev_consistency_step.argtypes = [I] * 6 + [P] * 6 + [ctypes.c_float] + [P] * 11 + [Z, P]
    nws = L.gradlev_consistency_workspace_bytes(2, 2, 100, 16, 16, 0)
    # the reverse scan's scratch with its own states, plus the forward's checkpoints
    assert nws >= L.gradlev_scan_workspace_bytes(2, 2, 100, 16, 16, 0, 1)
    assert L.gradlev_consistency_workspace_bytes(2, 2, 100, 16, 18, 0) == 0  # d_out % 4
    call = lambda v=fake, ws=fake, nbytes=1 << 30, d_out=16, dv=P(0): \
        L.gradlev_consistency_step(2, 2, 100, 16, d_out, 0, fake, fake, fake, fake, fake, v, 1.0,
                                   fake, fake, fake, fake, fake, fake, fake, fake, fake, dv, ws,
                                   nbytes, P(0))
    assert call(d_out=18) == 2           # d_out not a multiple of 4
    assert call(v=P(0)) == 1             # missing input
    assert call(v=P(4100)) == 1          # f32 v not 16-byte aligned
    assert call(dv=P(4100)) == 1
    assert call(ws=P(4096 + 16)) == 1    # workspace not 256-byte aligned
    assert call(nbytes=16) == 3          # workspace too small


def test_mlp2_recon_validates_before_launch(L):
    P = ctypes.c_void_p
    fake = P(4096)
    I, Z = ctypes.c_int, ctypes.c_size_t
    L.gradlev_mlp2_workspace_bytes.restype = Z
    L.gradlev_mlp2_workspace_bytes.argtypes = [I] * 7
    L.gradlev_mlp2_recon.restype = I
    L.gradlev_mlp2_recon.argtypes = [I] * 7 + [P] * 8 + [I] + [P] * 7 + [Z, P]
    assert L.gradlev_mlp2_workspace_bytes(2, 2, 64, 16, 32, 8, 0) > 0
    assert L.gradlev_mlp2_workspace_bytes(2, 2, 64, 16, 30, 8, 0) == 0   # d_h % 8
    assert L.gradlev_mlp2_workspace_bytes(2, 2, 64, 256, 128, 8, 0) == 0  # d_h * d_x too big
    call = lambda d_h=32, x=fake, ws=1 << 30, dW1=fake: L.gradlev_mlp2_recon(
        2, 2, 64, 16, d_h, 8, 0, x, fake, fake, fake, fake, fake, fake, fake, 0, fake, fake,
        fake, fake, fake, dW1, fake, ws, P(0))
    assert call(d_h=30) == 2
    assert call(x=P(0)) == 1
    assert call(dW1=P(4100)) == 1
    assert call(ws=16) == 3


def test_binding_refuses_host_tensors():
    """Host tensors never reach the library: its kernels would dereference them on the GPU."""
    torch = pytest.importorskip("torch")
    import token_weight_scans_b200 as tw
    B, H, T, d = 1, 1, 8, 16
    x = torch.zeros(B, H, T, d)
    gates = torch.zeros(B, H, T)
    W = torch.zeros(H, d, d)
    S = torch.zeros(B, H, d, d)
    calls = [
        lambda: tw.gradlev_scan_fwd(x, x, gates, gates, W),
        lambda: tw.gradlev_scan_bwd(x, x, gates, gates, W, x),
        lambda: tw.gradlev_scan_fwd_state(x, x, gates, gates, W, S),
        lambda: tw.gradlev_scan_bwd_state(x, x, gates, gates, W, x, S, S),
        lambda: tw.gradlev_decode_step(x, x, gates, gates, W, S),
        lambda: tw.gradlev_consistency_step(x, x, gates, gates, W, x),
        lambda: tw.gradlev_mlp2_recon(x, x, x, x, gates, gates, W, W),
    ]
    for c in calls:
        with pytest.raises(tw.GradlevError, match="CUDA device"):
            c()
