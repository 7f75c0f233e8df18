"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/sol.h declares, and rejects bad arguments before any
CUDA call (fake, never-dereferenced addresses are enough for that)."""
import ctypes
import os
import subprocess

import pytest

from video_diffusion_transformer_rms_b200 import _abi
from video_diffusion_transformer_rms_b200.build import LIB, build


@pytest.fixture(scope="module", autouse=True)
def built():
    build()


def test_header_declares_the_entry_points():
    syms = _abi.header_symbols()
    for name in ("sol_rms_adaln", "sol_gate_residual", "sol_qknorm_rope3d",
                 "sol_gate_residual_rms_adaln", "sol_residual_change",
                 "sol_residual_change_workspace_bytes", "sol_qknorm_rope3d_ex",
                 "sol_residual_change_noalloc", "sol_rope_table_bytes",
                 "sol_rope_table_build", "sol_qknorm_rope3d_tab", "sol_qknorm_rope3d_ex_tab",
                 "sol_status_string", "sol_last_error", "sol_version"):
        assert name in syms


def test_library_exports_every_declared_symbol():
    lib = _abi.lib()
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in _abi.header_symbols():
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings_and_version():
    assert _abi.status_string(_abi.SOL_OK) == "SOL_OK"
    assert _abi.status_string(_abi.SOL_ERR_MISALIGNED) == "SOL_ERR_MISALIGNED"
    assert _abi.status_string(99) == "SOL_ERR_UNKNOWN"
    assert _abi.sol_version() >> 16 == 2  # sol_qk_layout grew in 2.0
    assert _abi.sol_version() & 0xFFFF >= 1  # 2.1: the rotary table entry points


# Fake device addresses: validation must reject these calls on the host.
A = 0x7F0000000000
BF = _abi.SOL_BF16
F32 = _abi.SOL_F32


def rms(x=A, y=A + (1 << 30), sc=A + (2 << 30), sh=A + (3 << 30), g=None, B=1, L=4,
        nv=2, D=64, eps=1e-6, dt=BF):
    return _abi.sol_rms_adaln(x, y, sc, sh, g, B, L, nv, D, eps, dt, None)


def gate(h=A, br=A + (1 << 30), g=A + (2 << 30), out=A + (3 << 30), B=1, L=4, nv=2, D=64,
         dt=BF):
    return _abi.sol_gate_residual(h, br, g, out, B, L, nv, D, dt, None)


def qk(qkv=A, ldq=768, qo=A + (1 << 30), ko=A + (2 << 30), ldo=256, gq=None, gk=None, B=1,
       T=2, H=4, W=6, na=8, nh=2, hd=128, secs=(16, 24, 24), eps=1e-6, theta=1e4, dt=BF):
    return _abi.sol_qknorm_rope3d(qkv, ldq, qo, ko, ldo, gq, gk, B, T, H, W, na, nh, hd,
                                  *secs, eps, theta, dt, None)


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), _abi.SOL_ERR_INVALID_ARG),
    (dict(nv=5), _abi.SOL_ERR_INVALID_ARG),
    (dict(D=0), _abi.SOL_ERR_INVALID_ARG),
    (dict(eps=-1.0), _abi.SOL_ERR_INVALID_ARG),
    (dict(eps=float("nan")), _abi.SOL_ERR_INVALID_ARG),
    (dict(dt=7), _abi.SOL_ERR_INVALID_ARG),
    (dict(D=60), _abi.SOL_ERR_MISALIGNED),           # 120 bytes per row
    (dict(D=62, dt=F32), _abi.SOL_ERR_MISALIGNED),
    (dict(x=A + 8), _abi.SOL_ERR_MISALIGNED),
    (dict(g=A + (4 << 30) + 4), _abi.SOL_ERR_MISALIGNED),
    (dict(D=16392), _abi.SOL_ERR_UNSUPPORTED),
    (dict(D=8196, dt=F32), _abi.SOL_ERR_UNSUPPORTED),
    (dict(B=1 << 20, L=1 << 12), _abi.SOL_ERR_UNSUPPORTED),  # 2^32 rows
    (dict(B=1, L=1 << 31, nv=0), _abi.SOL_ERR_UNSUPPORTED),
    (dict(y=A + 16), _abi.SOL_ERR_INVALID_ARG),      # partial overlap with x
    (dict(y=A + (2 << 30) + 64), _abi.SOL_ERR_INVALID_ARG),  # overlaps scale
])
def test_rms_adaln_rejects(kw, status):
    assert rms(**kw) == status
    assert _abi.last_error() != ""


def test_zero_rows_is_a_noop_even_with_null_pointers():
    assert rms(x=None, y=None, B=0) == _abi.SOL_OK
    assert rms(x=None, y=None, L=0, nv=0) == _abi.SOL_OK
    assert gate(h=None, B=0) == _abi.SOL_OK
    assert qk(qkv=None, T=0, na=0) == _abi.SOL_OK
    assert _abi.last_error() == ""


@pytest.mark.parametrize("kw,status", [
    (dict(out=None), _abi.SOL_ERR_INVALID_ARG),
    (dict(nv=-1), _abi.SOL_ERR_INVALID_ARG),
    (dict(D=20), _abi.SOL_ERR_MISALIGNED),
    (dict(g=A + (2 << 30) + 2), _abi.SOL_ERR_MISALIGNED),
    (dict(D=16400), _abi.SOL_ERR_UNSUPPORTED),
    (dict(B=3, L=1 << 30, nv=0), _abi.SOL_ERR_UNSUPPORTED),
    (dict(out=A + 32), _abi.SOL_ERR_INVALID_ARG),     # partial overlap with h
    (dict(out=A + (1 << 30) - 32), _abi.SOL_ERR_INVALID_ARG),  # straddles branch
    (dict(out=A + (2 << 30)), _abi.SOL_ERR_INVALID_ARG),  # overlaps gate
])
def test_gate_residual_rejects(kw, status):
    assert gate(**kw) == status


def fused(h=A, br=A + (1 << 30), g=A + (2 << 30), ho=A + (3 << 30), y=A + (4 << 30),
          sc=A + (5 << 30), sh=A + (6 << 30), gm=None, B=1, L=4, nv=2, D=64, eps=1e-6, dt=BF):
    return _abi.sol_gate_residual_rms_adaln(h, br, g, ho, y, sc, sh, gm, B, L, nv, D, eps, dt,
                                            None)


@pytest.mark.parametrize("kw,status", [
    (dict(y=None), _abi.SOL_ERR_INVALID_ARG),
    (dict(sh=None), _abi.SOL_ERR_INVALID_ARG),
    (dict(nv=5), _abi.SOL_ERR_INVALID_ARG),
    (dict(eps=-1.0), _abi.SOL_ERR_INVALID_ARG),
    (dict(D=36), _abi.SOL_ERR_MISALIGNED),
    (dict(gm=A + (7 << 30) + 8), _abi.SOL_ERR_MISALIGNED),
    (dict(D=16392), _abi.SOL_ERR_UNSUPPORTED),
    (dict(B=1 << 20, L=1 << 12), _abi.SOL_ERR_UNSUPPORTED),
    (dict(ho=A + 64), _abi.SOL_ERR_INVALID_ARG),            # partial overlap with h
    (dict(ho=A + (1 << 30)), _abi.SOL_ERR_INVALID_ARG),     # h_out on branch
    (dict(y=A), _abi.SOL_ERR_INVALID_ARG),                  # y on h
    (dict(y=A + (3 << 30)), _abi.SOL_ERR_INVALID_ARG),      # y on h_out
    (dict(y=A + (5 << 30)), _abi.SOL_ERR_INVALID_ARG),      # y on scale
])
def test_gate_residual_rms_adaln_rejects(kw, status):
    assert fused(**kw) == status


def test_gate_residual_rms_adaln_zero_rows_noop():
    assert fused(h=None, y=None, B=0) == _abi.SOL_OK


def change(c=A, p=A + (1 << 30), po=None, B=2, L=4, D=64, out=A + (3 << 30),
           ws=A + (4 << 30), wsb=None, dt=BF):
    if wsb is None:
        wsb = _abi.sol_residual_change_workspace_bytes(B)
    return _abi.sol_residual_change(c, p, po, B, L, D, out, ws, wsb, dt, None)


def test_residual_change_workspace_size():
    assert _abi.sol_residual_change_workspace_bytes(0) == 0
    assert _abi.sol_residual_change_workspace_bytes(1) == 16384
    assert _abi.sol_residual_change_workspace_bytes(3) == 3 * 16384


@pytest.mark.parametrize("kw,status", [
    (dict(c=None), _abi.SOL_ERR_INVALID_ARG),
    (dict(out=None), _abi.SOL_ERR_INVALID_ARG),
    (dict(ws=None), _abi.SOL_ERR_INVALID_ARG),
    (dict(wsb=1000), _abi.SOL_ERR_INVALID_ARG),
    (dict(D=12), _abi.SOL_ERR_MISALIGNED),
    (dict(out=A + (3 << 30) + 4), _abi.SOL_ERR_MISALIGNED),
    (dict(ws=A + (4 << 30) + 8), _abi.SOL_ERR_MISALIGNED),
    (dict(B=70000, L=1), _abi.SOL_ERR_UNSUPPORTED),
    (dict(D=16400), _abi.SOL_ERR_UNSUPPORTED),
    (dict(po=A + 128), _abi.SOL_ERR_INVALID_ARG),           # prev_out overlaps cur
    (dict(po=A + (1 << 30) + 16), _abi.SOL_ERR_INVALID_ARG),  # partial overlap with prev
    (dict(out=A + 64), _abi.SOL_ERR_INVALID_ARG),           # out inside cur
    (dict(ws=A + (1 << 30)), _abi.SOL_ERR_INVALID_ARG),     # workspace on prev
    (dict(out=A + (4 << 30) + 64), _abi.SOL_ERR_INVALID_ARG),  # out inside workspace
])
def test_residual_change_rejects(kw, status):
    assert change(**kw) == status


def test_residual_change_zero_rows_noop():
    assert change(c=None, out=None, B=0) == _abi.SOL_OK
    assert change(c=None, L=0) == _abi.SOL_OK


@pytest.mark.parametrize("kw,status", [
    (dict(qkv=None), _abi.SOL_ERR_INVALID_ARG),
    (dict(hd=127, secs=(16, 24, 23)), _abi.SOL_ERR_INVALID_ARG),
    (dict(secs=(16, 24, 25)), _abi.SOL_ERR_INVALID_ARG),
    (dict(secs=(-1, 33, 32)), _abi.SOL_ERR_INVALID_ARG),
    (dict(theta=0.0), _abi.SOL_ERR_INVALID_ARG),
    (dict(ldq=500), _abi.SOL_ERR_INVALID_ARG),       # < 2*D
    (dict(ldo=200), _abi.SOL_ERR_INVALID_ARG),       # < D
    (dict(hd=96, secs=(16, 16, 16)), _abi.SOL_ERR_UNSUPPORTED),   # G = 12 lanes
    (dict(hd=8, secs=(2, 1, 1)), _abi.SOL_ERR_UNSUPPORTED),       # G = 1 lane (bf16)
    (dict(hd=256, secs=(32, 48, 48), dt=F32, ldq=1536, ldo=512),
     _abi.SOL_ERR_UNSUPPORTED),  # G = 64 lanes (fp32)
    (dict(nh=130, ldq=3 * 16640, ldo=16640), _abi.SOL_ERR_UNSUPPORTED),  # D > 16384
    (dict(T=1, H=1 << 16, W=1 << 16, na=0), _abi.SOL_ERR_UNSUPPORTED),  # H*W = 2^32
    (dict(T=0, H=1 << 16, W=1 << 16), _abi.SOL_ERR_UNSUPPORTED),
    (dict(B=1 << 22, T=1, H=32, W=32, na=0), _abi.SOL_ERR_UNSUPPORTED),  # 2^32 rows
    (dict(ldq=772), _abi.SOL_ERR_MISALIGNED),        # 1544-byte row stride
    (dict(qo=A + (1 << 30) + 2), _abi.SOL_ERR_MISALIGNED),
    (dict(qo=A + 512), _abi.SOL_ERR_INVALID_ARG),    # q_out inside qkv's k columns
    (dict(qo=A, ko=A + 1024, ldo=768), _abi.SOL_ERR_INVALID_ARG),  # half in place
    (dict(ko=A + (1 << 30) + 256, ldo=256), _abi.SOL_ERR_INVALID_ARG),  # q_out/k_out collide
])
def test_qknorm_rope3d_rejects(kw, status):
    assert qk(**kw) == status


def test_error_message_is_thread_local_and_cleared():
    assert rms(x=None) == _abi.SOL_ERR_INVALID_ARG
    msg = _abi.last_error()
    assert "non-null" in msg
    assert rms(B=0) == _abi.SOL_OK
    assert _abi.last_error() == ""


def test_python_binding_raises_with_reason():
    with pytest.raises(_abi.SolError) as ei:
        _abi.check(rms(D=60))
    assert ei.value.status == _abi.SOL_ERR_MISALIGNED
    assert "multiple of 16" in str(ei.value)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "_lib", None)
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "libsol.so"))
    with pytest.raises(ImportError):
        _abi.lib()
    assert isinstance(ctypes.CDLL, type)


# well-placed fp32 scale arrays for the INT8 cases (none overlaps another buffer)
Q8S, K8S, V8S = A + (3 << 30), A + (4 << 30), A + (6 << 30)


def qkex(qkv=A, ldq=3 * 1024, qo=A + (1 << 30), ko=A + (2 << 30), sb=None, sr=1024, sh=128,
         half=0, int8=0, qs=None, ks=None, B=1, T=2, H=4, W=6, na=8, nh=8, hd=128,
         secs=(16, 24, 24), dt=BF, per_axis=0, reserved=0, vo=None, vs=None):
    L = T * H * W + na
    lay = _abi.QkLayout(L * nh * hd if sb is None else sb, sr, sh, half, int8, qs, ks, per_axis,
                        reserved, vo, vs)
    return _abi.sol_qknorm_rope3d_ex(qkv, ldq, qo, ko, lay, None, None, B, T, H, W, na, nh, hd,
                                     *secs, 1e-6, 1e4, dt, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dt=F32), _abi.SOL_ERR_UNSUPPORTED),
    (dict(hd=32, secs=(4, 6, 6), nh=32), _abi.SOL_ERR_UNSUPPORTED),
    (dict(sr=-1), _abi.SOL_ERR_INVALID_ARG),
    (dict(sh=4), _abi.SOL_ERR_MISALIGNED),                      # 8-byte head stride
    (dict(qo=A + (1 << 30) + 8), _abi.SOL_ERR_MISALIGNED),
    (dict(int8=1), _abi.SOL_ERR_INVALID_ARG),                   # scales missing
    (dict(int8=1, qs=A + (3 << 30) + 2, ks=A + (4 << 30)), _abi.SOL_ERR_MISALIGNED),
    (dict(qo=A + 4096), _abi.SOL_ERR_INVALID_ARG),              # q_out inside qkv
    (dict(ko=A + (1 << 30) + 1024), _abi.SOL_ERR_INVALID_ARG),  # k_out overlaps q_out
    (dict(int8=1, qs=A + (1 << 30), ks=A + (4 << 30)), _abi.SOL_ERR_INVALID_ARG),  # scale on q
    (dict(reserved=1), _abi.SOL_ERR_INVALID_ARG),
    (dict(per_axis=2), _abi.SOL_ERR_INVALID_ARG),
    (dict(vo=A + (5 << 30)), _abi.SOL_ERR_UNSUPPORTED),          # v_out needs int8
    (dict(int8=1, qs=Q8S, ks=K8S, vo=A + (5 << 30)), _abi.SOL_ERR_INVALID_ARG),  # no v_scale
    (dict(int8=1, qs=Q8S, ks=K8S, vo=A + (5 << 30), vs=V8S, ldq=2 * 1024),
     _abi.SOL_ERR_INVALID_ARG),                                  # v not in the rows
    (dict(int8=1, qs=Q8S, ks=K8S, vo=A + (5 << 30) + 4, vs=V8S), _abi.SOL_ERR_MISALIGNED),
    (dict(int8=1, qs=Q8S, ks=K8S, vo=A + (5 << 30), vs=V8S + 2), _abi.SOL_ERR_MISALIGNED),
    (dict(int8=1, qs=Q8S, ks=K8S, vo=A + 4096, vs=V8S),
     _abi.SOL_ERR_INVALID_ARG),                                  # v_out on qkv's v columns
    (dict(int8=1, qs=Q8S, ks=K8S, vo=A + (2 << 30) + 64, vs=V8S),
     _abi.SOL_ERR_INVALID_ARG),                                  # v_out overlaps k_out
    (dict(int8=1, qs=Q8S, ks=K8S, vo=A + (5 << 30), vs=Q8S + 64),
     _abi.SOL_ERR_INVALID_ARG),                                  # v_scale overlaps q_scale
])
def test_qknorm_rope3d_ex_rejects(kw, status):
    assert qkex(**kw) == status


def test_qknorm_rope3d_ex_null_layout():
    assert _abi.sol_qknorm_rope3d_ex(A, 3 * 1024, A + (1 << 30), A + (2 << 30), None, None,
                                     None, 1, 2, 4, 6, 8, 8, 128, 16, 24, 24, 1e-6, 1e4, BF,
                                     None) == _abi.SOL_ERR_INVALID_ARG


# a fake table address far from every other fake buffer
TB = A + (8 << 30)


def table(data=TB, n_pos=8, hd=128, secs=(16, 24, 24), theta=1e4, per_axis=0):
    return _abi.RopeTable(data, n_pos, hd, *secs, theta, per_axis)


def test_rope_table_bytes():
    assert _abi.sol_rope_table_bytes(4680, 128) == 4680 * 128 * 4
    assert _abi.sol_rope_table_bytes(0, 128) == 0
    for n, hd in ((-1, 128), (10, 127), (10, 0), (10, 258), (1 << 31, 128)):
        assert _abi.sol_rope_table_bytes(n, hd) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(data=None), _abi.SOL_ERR_INVALID_ARG),
    (dict(data=TB + 4), _abi.SOL_ERR_MISALIGNED),
    (dict(n_pos=-1), _abi.SOL_ERR_INVALID_ARG),
    (dict(hd=127, secs=(16, 24, 23)), _abi.SOL_ERR_INVALID_ARG),
    (dict(hd=258, secs=(43, 43, 43)), _abi.SOL_ERR_INVALID_ARG),
    (dict(secs=(16, 24, 25)), _abi.SOL_ERR_INVALID_ARG),
    (dict(theta=0.0), _abi.SOL_ERR_INVALID_ARG),
    (dict(theta=float("nan")), _abi.SOL_ERR_INVALID_ARG),
    (dict(per_axis=2), _abi.SOL_ERR_INVALID_ARG),
])
def test_rope_table_build_rejects(kw, status):
    assert _abi.sol_rope_table_build(table(**kw), None) == status


def test_rope_table_build_null_and_empty():
    assert _abi.sol_rope_table_build(None, None) == _abi.SOL_ERR_INVALID_ARG
    assert _abi.sol_rope_table_build(table(n_pos=0), None) == _abi.SOL_OK


def qktab(tab=None, qkv=A, ldq=768, qo=A + (1 << 30), ko=A + (2 << 30), ldo=256, B=1, T=2,
          H=4, W=6, na=8, nh=2, dt=BF):
    tab = table() if tab is None else tab
    return _abi.sol_qknorm_rope3d_tab(qkv, ldq, qo, ko, ldo, None, None, tab, B, T, H, W, na,
                                      nh, 1e-6, dt, None)


@pytest.mark.parametrize("kw,status", [
    (dict(tab=table(n_pos=7)), _abi.SOL_ERR_INVALID_ARG),     # needs max(T, H, W, na) = 8
    (dict(tab=table(data=None)), _abi.SOL_ERR_INVALID_ARG),
    (dict(tab=table(data=TB + 8)), _abi.SOL_ERR_MISALIGNED),
    (dict(tab=table(secs=(16, 24, 25))), _abi.SOL_ERR_INVALID_ARG),
    (dict(tab=table(data=A + (1 << 30) + 4096)), _abi.SOL_ERR_INVALID_ARG),  # table under q_out
    (dict(tab=table(data=A + (2 << 30))), _abi.SOL_ERR_INVALID_ARG),         # ... under k_out
    (dict(qkv=None), _abi.SOL_ERR_INVALID_ARG),                # the usual checks still apply
    (dict(ldo=200), _abi.SOL_ERR_INVALID_ARG),
    (dict(qo=A + 512), _abi.SOL_ERR_INVALID_ARG),
    (dict(T=1, H=1 << 16, W=1 << 16, na=0), _abi.SOL_ERR_UNSUPPORTED),
])
def test_qknorm_rope3d_tab_rejects(kw, status):
    assert qktab(**kw) == status


def test_qknorm_rope3d_tab_positions_needed():
    # video-only calls need max(T, H, W) rows, audio-only calls n_audio rows
    assert qktab(tab=table(n_pos=4), T=3, H=5, W=4, na=0) == _abi.SOL_ERR_INVALID_ARG
    assert qktab(tab=table(n_pos=10), T=0, H=0, W=0, na=11) == _abi.SOL_ERR_INVALID_ARG
    assert "positions" in _abi.last_error()
    # zero rows: nothing to check against the table's size
    assert qktab(tab=table(n_pos=0), B=0) == _abi.SOL_OK


def qkextab(tab=None, per_axis=0, int8=0, qs=None, ks=None, **kw):
    tab = table() if tab is None else tab
    L = 2 * 4 * 6 + 8
    nh, hd = 8, 128
    lay = _abi.QkLayout(L * nh * hd, nh * hd, hd, 0, int8, qs, ks, per_axis, 0, None, None)
    return _abi.sol_qknorm_rope3d_ex_tab(A, 3 * 1024, A + (1 << 30), A + (2 << 30), lay, None,
                                         None, tab, 1, 2, 4, 6, 8, nh, 1e-6, BF, None)


def test_qknorm_rope3d_ex_tab_rejects():
    # the layout's frequency rule must be the table's
    assert qkextab(per_axis=1) == _abi.SOL_ERR_INVALID_ARG
    assert "per_axis_freq" in _abi.last_error()
    assert qkextab(tab=table(per_axis=1)) == _abi.SOL_ERR_INVALID_ARG
    assert qkextab(tab=table(n_pos=7)) == _abi.SOL_ERR_INVALID_ARG
    # a scale array over the table
    assert qkextab(int8=1, qs=TB + 256, ks=Q8S) == _abi.SOL_ERR_INVALID_ARG
    assert _abi.sol_qknorm_rope3d_ex_tab(A, 3 * 1024, A + (1 << 30), A + (2 << 30), None, None,
                                         None, table(), 1, 2, 4, 6, 8, 8, 1e-6, BF,
                                         None) == _abi.SOL_ERR_INVALID_ARG
    assert _abi.sol_qknorm_rope3d_ex_tab(A, 3 * 1024, A + (1 << 30), A + (2 << 30), None, None,
                                         None, None, 1, 2, 4, 6, 8, 8, 1e-6, BF,
                                         None) == _abi.SOL_ERR_INVALID_ARG


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "sol.h"

int main(void) {
    sol_qk_layout lay;
    memset(&lay, 0, sizeof lay);
    lay.stride_b = 1;
    lay.stride_row = 1;
    lay.stride_head = 1;
    lay.reserved = 1; /* must be 0: refused before any CUDA call */
    if ((sol_version() >> 16) != 2) return 1;
    if (sol_rms_adaln(NULL, NULL, NULL, NULL, NULL, 1, 4, 4, 8, 1e-6f, SOL_BF16, NULL) !=
        SOL_ERR_INVALID_ARG) return 2;
    if (strlen(sol_last_error()) == 0) return 3;
    if (sol_qknorm_rope3d_ex((const void *)0x1000, 3 * 256, (void *)0x100000,
                             (void *)0x200000, &lay, NULL, NULL, 1, 2, 4, 6, 8, 2, 128,
                             16, 24, 24, 1e-6f, 1e4f, SOL_BF16, NULL) != SOL_ERR_INVALID_ARG)
        return 4;
    printf("%s | %s\n", sol_status_string(SOL_ERR_INVALID_ARG), sol_last_error());
    return 0;
}
"""


def test_header_is_plain_c_and_the_library_links_from_c(tmp_path):
    # the boundary is a C ABI: a C99 client compiles against include/sol.h with
    # every warning an error, links libsol.so and gets statuses back (no GPU
    # call is made: both calls fail validation)
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(_abi.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(root, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-lsol", f"-Wl,-rpath,{libdir}"], check=True)
    p = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert p.returncode == 0, (p.returncode, p.stdout, p.stderr)
    assert "layout.reserved must be 0" in p.stdout


def test_cutlass_tree_is_explicit(monkeypatch, tmp_path):
    # the GEMM + GELU kernel names its CUTLASS tree: SOL_CUTLASS_DIR when set,
    # else the copy vendored in flashinfer; a missing or old tree fails with
    # the path in the message
    from video_diffusion_transformer_rms_b200 import build as b
    root, ver = b.cutlass_info()
    assert tuple(int(x) for x in ver.split("."))[:2] >= b.CUTLASS_MIN
    monkeypatch.setenv("SOL_CUTLASS_DIR", str(tmp_path))
    with pytest.raises(RuntimeError, match="SOL_CUTLASS_DIR"):
        b.cutlass_info()
    inc = tmp_path / "include"
    (inc / "cute").mkdir(parents=True)
    (inc / "cutlass").mkdir()
    (inc / "cutlass" / "version.h").write_text(
        "#define CUTLASS_MAJOR 4\n#define CUTLASS_MINOR 5\n#define CUTLASS_PATCH 1\n")
    assert b.cutlass_info() == (str(tmp_path), "4.5.1")
    (inc / "cutlass" / "version.h").write_text(
        "#define CUTLASS_MAJOR 3\n#define CUTLASS_MINOR 5\n#define CUTLASS_PATCH 0\n")
    with pytest.raises(RuntimeError, match="version"):
        b.cutlass_info()
