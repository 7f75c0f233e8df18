"""GPU parity: the CUDA kernels (called through the C ABI) against the fp64
oracle on the same seeded inputs, element by element, within
|gpu - oracle| <= 2 ulp(oracle value) + 1e-3.

Small workloads are compared in full; the 5 s / 15 s clip shapes and the CFG
batch are compared on a seeded sample of rows (always including each
sample's first/last rows and its video/audio boundary) at full size, in the
launch configuration the benchmark uses.  Edge cases: ragged widths and row
counts, no audio / no video, in-place outputs, strided layouts, guard bytes
around outputs, zero rows, misaligned pointers.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import assert_close, sample_rows, take_rows, take_rows_gpu
from video_diffusion_transformer_rms_b200 import _abi, api
from video_diffusion_transformer_rms_b200.workloads import (WORKLOADS, activation,
                                                            make_inputs, to_oracle_array,
                                                            vectors)

pytestmark = pytest.mark.gpu
DEV = "cuda"
SMALL = ("tiny", "medium")
LARGE = ("clip5s", "clip15s", "cfg5s", "cfg5s_d3072")


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    _abi.lib()
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _ids(w, n=1024):
    return sample_rows(w.rows, w.L, w.n_video, w.B, n, seed=7 + w.index)


def _o(t):
    return to_oracle_array(t)


# ----------------------------------------------------------------------------
# RMS-AdaLN
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("name", SMALL + LARGE)
@pytest.mark.parametrize("with_gamma", [False, True])
def test_rms_adaln_workload(name, with_gamma):
    w = WORKLOADS[name]
    t = make_inputs(w, DEV, which=("rms_adaln",), with_gamma=with_gamma)
    x = t["x"].view(w.B, w.L, w.D)
    y = api.rms_adaln(x, t["scale"], t["shift"], w.n_video, gamma=t.get("gamma"), eps=w.eps)
    torch.cuda.synchronize()
    x2, y2 = x.view(w.rows, w.D), y.view(w.rows, w.D)
    g = _o(t["gamma"]) if with_gamma else None
    if name in SMALL:
        want = oracle.rms_adaln(_o(x2), _o(t["scale"]), _o(t["shift"]), w.L, w.n_video,
                                w.eps, gamma=g)
        assert_close(y2, want, f"rms_adaln[{name}]")
    else:
        ids = _ids(w)
        want = oracle.rms_adaln(take_rows(x2, ids), _o(t["scale"]), _o(t["shift"]), w.L,
                                w.n_video, w.eps, gamma=g, row_ids=ids)
        assert_close(take_rows_gpu(y2, ids), want, f"rms_adaln[{name}] sampled")


RMS_SHAPES = [
    # B, L, n_video, D, dtype
    (1, 1, 1, 8, torch.bfloat16),            # one vector per row, one row
    (3, 37, 20, 5128, torch.bfloat16),       # ragged: 641 vectors per row
    (2, 300, 0, 4096, torch.bfloat16),       # audio only
    (2, 300, 300, 2056, torch.bfloat16),     # video only, ragged
    (1, 1000, 500, 256, torch.float32),
    (1, 33, 16, 16384, torch.bfloat16),      # widest bf16 row
    (1, 17, 5, 8192, torch.float32),         # widest fp32 row
    (5, 1000, 900, 3072, torch.bfloat16),
    (1, 50001, 49000, 128, torch.bfloat16),  # many more rows than CTAs
    (1, 7, 3, 12, torch.float32),            # 3 vectors per row
]


def _rand_rms(B, L, D, dt, seed):
    x = activation(B * L, D, dt, DEV, seed, outliers=True).view(B, L, D)
    sc = vectors((B, 2, D), 0.0, 0.5, dt, DEV, seed + 1)
    sh = vectors((B, 2, D), 0.0, 0.5, dt, DEV, seed + 2)
    g = vectors((D,), 1.0, 0.1, dt, DEV, seed + 3)
    return x, sc, sh, g


@pytest.mark.parametrize("B,L,nv,D,dt", RMS_SHAPES)
def test_rms_adaln_shapes(B, L, nv, D, dt):
    x, sc, sh, g = _rand_rms(B, L, D, dt, seed=D + L)
    for gamma in (None, g):
        y = api.rms_adaln(x, sc, sh, nv, gamma=gamma, eps=1e-6)
        want = oracle.rms_adaln(_o(x.view(-1, D)), _o(sc), _o(sh), L, nv, 1e-6,
                                gamma=None if gamma is None else _o(g))
        assert_close(y.view(-1, D), want, f"rms_adaln B={B} L={L} D={D}")


def test_rms_adaln_in_place_and_guards():
    B, L, nv, D = 2, 777, 700, 5120
    x, sc, sh, _ = _rand_rms(B, L, D, torch.bfloat16, seed=3)
    want = oracle.rms_adaln(_o(x.view(-1, D)), _o(sc), _o(sh), L, nv, 1e-6)
    # in place
    xi = x.clone()
    api.rms_adaln(xi, sc, sh, nv, out=xi)
    assert_close(xi.view(-1, D), want, "rms_adaln in place")
    # output inside a guarded buffer: the 4 KB on each side must stay intact
    pad = 2048
    buf = torch.full((B * L * D + 2 * pad,), 7.0, dtype=torch.bfloat16, device=DEV)
    y = buf[pad:pad + B * L * D].view(B, L, D)
    api.rms_adaln(x, sc, sh, nv, out=y)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == 7.0) and torch.all(buf[-pad:] == 7.0)
    assert_close(y.view(-1, D), want, "rms_adaln guarded")


def test_rms_adaln_zero_rows_touch_nothing():
    D = 256
    x = torch.zeros((0, 5, D), dtype=torch.bfloat16, device=DEV)
    y = torch.full((1, 5, D), 3.0, dtype=torch.bfloat16, device=DEV)
    sc = torch.zeros((1, 2, D), dtype=torch.bfloat16, device=DEV)
    st = _abi.sol_rms_adaln(x.data_ptr(), y.data_ptr(), sc.data_ptr(), sc.data_ptr(), None,
                            0, 5, 2, D, 1e-6, _abi.SOL_BF16, None)
    assert st == _abi.SOL_OK
    torch.cuda.synchronize()
    assert torch.all(y == 3.0)


def test_rms_adaln_misaligned_is_rejected_without_writing():
    D = 64
    x = torch.randn((1, 4, D), device=DEV).to(torch.bfloat16)
    y = torch.full((4 * D + 8,), 5.0, dtype=torch.bfloat16, device=DEV)
    sc = torch.zeros((1, 2, D), dtype=torch.bfloat16, device=DEV)
    st = _abi.sol_rms_adaln(x.data_ptr(), y.data_ptr() + 2, sc.data_ptr(), sc.data_ptr(), None,
                            1, 4, 2, D, 1e-6, _abi.SOL_BF16, None)
    assert st == _abi.SOL_ERR_MISALIGNED
    torch.cuda.synchronize()
    assert torch.all(y == 5.0)


def test_rms_adaln_is_deterministic():
    w = WORKLOADS["medium"]
    t = make_inputs(w, DEV, which=("rms_adaln",))
    x = t["x"].view(w.B, w.L, w.D)
    y1 = api.rms_adaln(x, t["scale"], t["shift"], w.n_video)
    y2 = api.rms_adaln(x, t["scale"], t["shift"], w.n_video)
    assert torch.equal(y1, y2)


# ----------------------------------------------------------------------------
# Gated residual
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("name", SMALL + LARGE)
def test_gate_residual_workload(name):
    w = WORKLOADS[name]
    t = make_inputs(w, DEV, which=("gate_residual",))
    h, br = t["h"].view(w.B, w.L, w.D), t["branch"].view(w.B, w.L, w.D)
    out = api.gate_residual(h, br, t["gate"], w.n_video)
    torch.cuda.synchronize()
    h2, b2, o2 = h.view(-1, w.D), br.view(-1, w.D), out.view(-1, w.D)
    if name in SMALL:
        want = oracle.gate_residual(_o(h2), _o(b2), _o(t["gate"]), w.L, w.n_video)
        assert_close(o2, want, f"gate_residual[{name}]")
    else:
        ids = _ids(w)
        want = oracle.gate_residual(take_rows(h2, ids), take_rows(b2, ids), _o(t["gate"]),
                                    w.L, w.n_video, row_ids=ids)
        assert_close(take_rows_gpu(o2, ids), want, f"gate_residual[{name}] sampled")


@pytest.mark.parametrize("B,L,nv,D,dt", RMS_SHAPES)
def test_gate_residual_shapes(B, L, nv, D, dt):
    h = activation(B * L, D, dt, DEV, 11, outliers=True).view(B, L, D)
    br = activation(B * L, D, dt, DEV, 12, outliers=True).view(B, L, D)
    g = vectors((B, 2, D), 0.0, 0.1, dt, DEV, 13)
    out = api.gate_residual(h, br, g, nv)
    want = oracle.gate_residual(_o(h.view(-1, D)), _o(br.view(-1, D)), _o(g), L, nv)
    assert_close(out.view(-1, D), want, f"gate_residual B={B} L={L} D={D}")


def test_gate_residual_in_place_zero_gate_and_guards():
    B, L, nv, D = 2, 513, 500, 3072
    dt = torch.bfloat16
    h = activation(B * L, D, dt, DEV, 21, outliers=True).view(B, L, D)
    br = activation(B * L, D, dt, DEV, 22, outliers=True).view(B, L, D)
    g = vectors((B, 2, D), 0.0, 0.1, dt, DEV, 23)
    want = oracle.gate_residual(_o(h.view(-1, D)), _o(br.view(-1, D)), _o(g), L, nv)
    for which in ("h", "branch"):
        hi, bi = h.clone(), br.clone()
        api.gate_residual(hi, bi, g, nv, out=hi if which == "h" else bi)
        assert_close((hi if which == "h" else bi).view(-1, D), want, f"in place on {which}")
    # gate = 0 returns h bit for bit
    z = torch.zeros_like(g)
    assert torch.equal(api.gate_residual(h, br, z, nv), h)
    pad = 4096
    buf = torch.full((B * L * D + 2 * pad,), -9.0, dtype=dt, device=DEV)
    o = buf[pad:pad + B * L * D].view(B, L, D)
    api.gate_residual(h, br, g, nv, out=o)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == -9.0) and torch.all(buf[-pad:] == -9.0)
    assert_close(o.view(-1, D), want, "gate_residual guarded")


# ----------------------------------------------------------------------------
# Fused gated residual + RMS-AdaLN
# ----------------------------------------------------------------------------

def _check_fused(h2, b2, gate, sc, sh, L, nv, eps, gamma, ho2, y2, what, ids=None):
    if ids is None:
        wh, wy = oracle.gate_residual_rms_adaln(_o(h2), _o(b2), _o(gate), _o(sc), _o(sh), L, nv,
                                                eps, gamma=None if gamma is None else _o(gamma))
        assert_close(ho2, wh, f"{what} h_out")
        assert_close(y2, wy, f"{what} y")
    else:
        wh, wy = oracle.gate_residual_rms_adaln(take_rows(h2, ids), take_rows(b2, ids), _o(gate),
                                                _o(sc), _o(sh), L, nv, eps,
                                                gamma=None if gamma is None else _o(gamma),
                                                row_ids=ids)
        assert_close(take_rows_gpu(ho2, ids), wh, f"{what} h_out sampled")
        assert_close(take_rows_gpu(y2, ids), wy, f"{what} y sampled")


@pytest.mark.parametrize("name", SMALL + ("clip5s", "cfg5s", "cfg5s_d3072"))
@pytest.mark.parametrize("with_gamma", [False, True])
def test_gate_residual_rms_adaln_workload(name, with_gamma):
    w = WORKLOADS[name]
    t = make_inputs(w, DEV, which=("rms_adaln", "gate_residual"), with_gamma=with_gamma)
    h, br = t["h"].view(w.B, w.L, w.D), t["branch"].view(w.B, w.L, w.D)
    gamma = t.get("gamma")
    ho, y = api.gate_residual_rms_adaln(h, br, t["gate"], t["scale"], t["shift"], w.n_video,
                                        gamma=gamma, eps=w.eps)
    torch.cuda.synchronize()
    ids = None if name in SMALL else _ids(w)
    _check_fused(h.view(-1, w.D), br.view(-1, w.D), t["gate"], t["scale"], t["shift"], w.L,
                 w.n_video, w.eps, gamma, ho.view(-1, w.D), y.view(-1, w.D), f"fused[{name}]",
                 ids)


@pytest.mark.parametrize("B,L,nv,D,dt", RMS_SHAPES)
def test_gate_residual_rms_adaln_shapes(B, L, nv, D, dt):
    h = activation(B * L, D, dt, DEV, 41, outliers=True).view(B, L, D)
    br = activation(B * L, D, dt, DEV, 42, outliers=True).view(B, L, D)
    g = vectors((B, 2, D), 0.0, 0.1, dt, DEV, 43)
    _, sc, sh, gm = _rand_rms(1, 1, D, dt, seed=44)
    sc = vectors((B, 2, D), 0.0, 0.5, dt, DEV, 45)
    sh = vectors((B, 2, D), 0.0, 0.5, dt, DEV, 46)
    for gamma in (None, gm):
        ho, y = api.gate_residual_rms_adaln(h, br, g, sc, sh, nv, gamma=gamma)
        _check_fused(h.view(-1, D), br.view(-1, D), g, sc, sh, L, nv, 1e-6, gamma,
                     ho.view(-1, D), y.view(-1, D), f"fused B={B} L={L} D={D}")


def test_gate_residual_rms_adaln_in_place_and_guards():
    B, L, nv, D = 2, 601, 555, 5120
    dt = torch.bfloat16
    h = activation(B * L, D, dt, DEV, 51, outliers=True).view(B, L, D)
    br = activation(B * L, D, dt, DEV, 52, outliers=True).view(B, L, D)
    g = vectors((B, 2, D), 0.0, 0.1, dt, DEV, 53)
    sc = vectors((B, 2, D), 0.0, 0.5, dt, DEV, 54)
    sh = vectors((B, 2, D), 0.0, 0.5, dt, DEV, 55)
    wh, wy = oracle.gate_residual_rms_adaln(_o(h.view(-1, D)), _o(br.view(-1, D)), _o(g), _o(sc),
                                            _o(sh), L, nv, 1e-6)
    # residual stream updated in place
    hi = h.clone()
    _, y = api.gate_residual_rms_adaln(hi, br, g, sc, sh, nv, h_out=hi)
    assert_close(hi.view(-1, D), wh, "fused in place h_out")
    assert_close(y.view(-1, D), wy, "fused in place y")
    # outputs inside guarded buffers
    pad = 4096
    n = B * L * D
    bh = torch.full((n + 2 * pad,), 3.0, dtype=dt, device=DEV)
    by = torch.full((n + 2 * pad,), -3.0, dtype=dt, device=DEV)
    ho, y = api.gate_residual_rms_adaln(h, br, g, sc, sh, nv, h_out=bh[pad:pad + n].view(B, L, D),
                                        y=by[pad:pad + n].view(B, L, D))
    torch.cuda.synchronize()
    assert torch.all(bh[:pad] == 3.0) and torch.all(bh[-pad:] == 3.0)
    assert torch.all(by[:pad] == -3.0) and torch.all(by[-pad:] == -3.0)
    assert_close(ho.view(-1, D), wh, "fused guarded h_out")
    assert_close(y.view(-1, D), wy, "fused guarded y")
    # gate = 0: h_out is h bit for bit and y equals sol_rms_adaln(h)
    z = torch.zeros_like(g)
    ho, y = api.gate_residual_rms_adaln(h, br, z, sc, sh, nv)
    assert torch.equal(ho, h)
    assert torch.equal(y, api.rms_adaln(h, sc, sh, nv))


# ----------------------------------------------------------------------------
# First-Block-Cache change detector
# ----------------------------------------------------------------------------

def _change_close(got, want, what):
    """Relative error <= 1e-5 on num, den and rel (fp32 row partials of at most
    64 terms, fp64 beyond); exact zeros and infinities must match."""
    g = got.detach().cpu().numpy()
    assert g.shape == want.shape, what
    inf = np.isinf(want)
    assert np.array_equal(np.isinf(g), inf), what
    fin = ~inf
    np.testing.assert_allclose(g[fin], want[fin], rtol=1e-5, atol=1e-30, err_msg=what)


def _next_step(prev, rel_noise, seed):
    """A 'next step' residual: prev plus relative noise (a few percent)."""
    g = torch.Generator(device=prev.device).manual_seed(seed)
    n = torch.randn(prev.shape, generator=g, device=prev.device, dtype=torch.float32)
    return (prev.float() * (1.0 + rel_noise * n)).to(prev.dtype)


@pytest.mark.parametrize("name", SMALL + ("clip5s", "clip15s", "cfg5s", "cfg5s_d3072"))
def test_residual_change_workload(name):
    w = WORKLOADS[name]
    prev = activation(w.rows, w.D, w.torch_dtype, DEV, seed_for_change(w), w.outliers)
    cur = _next_step(prev, 0.05, 7)
    out = api.residual_change(cur.view(w.B, w.L, w.D), prev.view(w.B, w.L, w.D))
    want = oracle.residual_change(_o(cur), _o(prev), w.B, w.L)
    _change_close(out, want, f"residual_change[{name}]")
    assert 0.01 < want[-1, 2] < 0.2


def seed_for_change(w):
    return 77_000 + w.index


RC_SHAPES = [
    (1, 1, 8, torch.bfloat16), (3, 37, 5128, torch.bfloat16), (2, 1000, 256, torch.float32),
    (5, 999, 3072, torch.bfloat16), (1, 33, 16384, torch.bfloat16), (2, 17, 8192, torch.float32),
    (70, 3, 512, torch.bfloat16), (1, 50001, 128, torch.bfloat16),
]


@pytest.mark.parametrize("B,L,D,dt", RC_SHAPES)
def test_residual_change_shapes(B, L, D, dt):
    prev = activation(B * L, D, dt, DEV, 91, outliers=True)
    cur = _next_step(prev, 0.1, 92)
    out = api.residual_change(cur.view(B, L, D), prev.view(B, L, D))
    _change_close(out, oracle.residual_change(_o(cur), _o(prev), B, L), f"rc B={B} L={L} D={D}")


def test_residual_change_refresh_zero_and_determinism():
    B, L, D, dt = 2, 3001, 5120, torch.bfloat16
    prev = activation(B * L, D, dt, DEV, 93, outliers=True).view(B, L, D)
    cur = _next_step(prev, 0.03, 94)
    want = oracle.residual_change(_o(cur.view(-1, D)), _o(prev.view(-1, D)), B, L)
    # cache refresh into a separate, guarded buffer
    pad = 4096
    n = B * L * D
    buf = torch.full((n + 2 * pad,), 9.0, dtype=dt, device=DEV)
    po = buf[pad:pad + n].view(B, L, D)
    out = api.residual_change(cur, prev, prev_out=po)
    torch.cuda.synchronize()
    assert torch.equal(po, cur)
    assert torch.all(buf[:pad] == 9.0) and torch.all(buf[-pad:] == 9.0)
    _change_close(out, want, "rc refresh")
    # refresh in place over prev; then the next comparison sees no change
    p2 = prev.clone()
    out = api.residual_change(cur, p2, prev_out=p2)
    _change_close(out, want, "rc in-place refresh")
    assert torch.equal(p2, cur)
    out = api.residual_change(cur, p2)
    assert torch.all(out[:, 0] == 0) and torch.all(out[:, 2] == 0)
    # zero previous residual: rel is +inf where anything changed, 0 otherwise
    z = torch.zeros_like(prev)
    out = api.residual_change(cur, z)
    assert torch.all(torch.isinf(out[:, 2]))
    out = api.residual_change(z, z)
    assert torch.all(out == 0)
    # deterministic: same bits on every call
    ws = torch.empty(_abi.sol_residual_change_workspace_bytes(B), dtype=torch.uint8, device=DEV)
    a = api.residual_change(cur, prev, workspace=ws)
    b = api.residual_change(cur, prev, workspace=ws)
    assert torch.equal(a, b)


# ----------------------------------------------------------------------------
# QKNorm + 3D RoPE
# ----------------------------------------------------------------------------

def _qk_oracle(qkv2, w_like, gq, gk, ids=None):
    T, H, W, na, nh, hd, secs, eps, theta = w_like
    return oracle.qknorm_rope3d(qkv2, T, H, W, na, nh, hd, secs, eps, theta,
                                gamma_q=gq, gamma_k=gk, row_ids=ids)


def _table(use, T, H, W, na, hd, secs=(16, 24, 24), theta=1e4, per_axis=False):
    """The rotary table of the table-driven entry points (sol_qknorm_rope3d_tab,
    sol_qknorm_rope3d_ex_tab) covering a call's positions, or None for the
    on-the-fly ones."""
    if not use:
        return None
    return api.RopeTable.for_grid(T, H, W, na, hd, sections=secs, theta=theta,
                                  per_axis_freq=per_axis, device=DEV)


ROPE = pytest.mark.parametrize("tab", [False, True], ids=["otf", "table"])


@pytest.mark.parametrize("name", SMALL + LARGE)
@ROPE
def test_qknorm_rope3d_workload(name, tab):
    w = WORKLOADS[name]
    t = make_inputs(w, DEV, which=("qknorm_rope3d",))
    qkv = t["qkv"].view(w.B, w.L, 3 * w.D)
    q, k = api.qknorm_rope3d(qkv, w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim,
                             w.sections, t["gamma_q"], t["gamma_k"], w.eps, w.theta,
                             table=_table(tab, w.T, w.H, w.W, w.n_audio, w.head_dim, w.sections,
                                          w.theta))
    torch.cuda.synchronize()
    spec = (w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim, w.sections, w.eps, w.theta)
    q2, k2 = q.reshape(-1, w.D), k.reshape(-1, w.D)
    qkv2 = qkv.view(-1, 3 * w.D)
    gq, gk = _o(t["gamma_q"]), _o(t["gamma_k"])
    if name in SMALL:
        wq, wk = _qk_oracle(_o(qkv2), spec, gq, gk)
        assert_close(q2, wq, f"q[{name}]")
        assert_close(k2, wk, f"k[{name}]")
    else:
        ids = _ids(w, 512)
        wq, wk = _qk_oracle(take_rows(qkv2[:, :2 * w.D], ids), spec, gq, gk, ids)
        assert_close(take_rows_gpu(q2, ids), wq, f"q[{name}] sampled")
        assert_close(take_rows_gpu(k2, ids), wk, f"k[{name}] sampled")


QK_CASES = [
    # B, T, H, W, n_audio, n_heads, head_dim, sections, dtype, pad
    (1, 2, 4, 6, 8, 2, 128, (16, 24, 24), torch.float32, 0),
    (1, 2, 4, 6, 8, 3, 64, (8, 12, 12), torch.float32, 4),       # G = 16 lanes
    (2, 3, 5, 7, 11, 5, 64, (8, 12, 12), torch.bfloat16, 8),     # G = 8, padded rows
    (1, 2, 3, 4, 5, 3, 256, (32, 48, 48), torch.bfloat16, 0),    # G = 32
    (1, 2, 2, 2, 3, 4, 32, (4, 6, 6), torch.bfloat16, 0),        # G = 4
    (1, 1, 2, 2, 1, 2, 16, (2, 3, 3), torch.bfloat16, 0),        # G = 2
    (3, 1, 1, 1, 0, 40, 128, (16, 24, 24), torch.bfloat16, 0),   # one video row, no audio
    (2, 0, 0, 0, 300, 8, 128, (16, 24, 24), torch.bfloat16, 0),  # audio only
    (1, 4, 9, 13, 0, 24, 128, (16, 24, 24), torch.bfloat16, 0),  # video only
    (1, 2, 4, 6, 8, 41, 128, (16, 24, 24), torch.bfloat16, 0),   # ragged thread tail
    (1, 2, 4, 6, 9, 128, 128, (16, 24, 24), torch.bfloat16, 0),  # widest row, D=16384
    (1, 3, 4, 5, 7, 4, 128, (64, 0, 0), torch.bfloat16, 0),      # 1D RoPE (t only)
    (1, 10, 40, 50, 1000, 8, 128, (16, 24, 24), torch.bfloat16, 8),  # many rows
    (3, 3, 7, 11, 500, 40, 128, (16, 24, 24), torch.bfloat16, 16),   # CTAs cross W, H,
    # video/audio and sample boundaries inside their row share
]


@pytest.mark.parametrize("B,T,H,W,na,nh,hd,secs,dt,pad", QK_CASES)
@ROPE
def test_qknorm_rope3d_cases(B, T, H, W, na, nh, hd, secs, dt, pad, tab):
    D = nh * hd
    L = T * H * W + na
    C = 3 * D + pad
    qkv = activation(B * L, C, dt, DEV, 31 + hd, outliers=True).view(B, L, C)
    gq = vectors((hd,), 1.0, 0.1, dt, DEV, 32)
    gk = vectors((hd,), 1.0, 0.1, dt, DEV, 33)
    spec = (T, H, W, na, nh, hd, secs, 1e-6, 1e4)
    table = _table(tab, T, H, W, na, hd, secs)
    for gam in ((gq, gk), (None, None)):
        q, k = api.qknorm_rope3d(qkv, T, H, W, na, nh, hd, secs, gam[0], gam[1], table=table)
        wq, wk = _qk_oracle(_o(qkv.view(B * L, C)), spec,
                            None if gam[0] is None else _o(gq),
                            None if gam[1] is None else _o(gk))
        assert_close(q.reshape(-1, D), wq, "q")
        assert_close(k.reshape(-1, D), wk, "k")


@ROPE
def test_qknorm_rope3d_layouts_and_v_untouched(tab):
    w = WORKLOADS["medium"]
    D = w.D
    t = make_inputs(w, DEV, which=("qknorm_rope3d",))
    qkv = t["qkv"].view(w.B, w.L, 3 * D)
    args = (w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim, w.sections, t["gamma_q"],
            t["gamma_k"])
    table = _table(tab, w.T, w.H, w.W, w.n_audio, w.head_dim)
    kw = {"table": table}
    spec = (w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim, w.sections, w.eps, w.theta)
    ids = sample_rows(w.rows, w.L, w.n_video, w.B, 1500, seed=5)
    wq, wk = _qk_oracle(take_rows(qkv.view(-1, 3 * D)[:, :2 * D], ids), spec,
                        _o(t["gamma_q"]), _o(t["gamma_k"]), ids)
    # separate q and k tensors (ld_out = D)
    qo = torch.empty((w.B, w.L, D), dtype=qkv.dtype, device=DEV)
    ko = torch.empty_like(qo)
    api.qknorm_rope3d(qkv, *args, q_out=qo, k_out=ko, **kw)
    assert_close(take_rows_gpu(qo.view(-1, D), ids), wq, "q separate")
    assert_close(take_rows_gpu(ko.view(-1, D), ids), wk, "k separate")
    # in place, v columns untouched
    qi = qkv.clone()
    v_before = qi[..., 2 * D:].clone()
    api.qknorm_rope3d(qi, *args, q_out=qi[..., :D], k_out=qi[..., D:2 * D], **kw)
    torch.cuda.synchronize()
    assert torch.equal(qi[..., 2 * D:], v_before)
    assert_close(take_rows_gpu(qi.view(-1, 3 * D)[:, :D], ids), wq, "q in place")
    assert_close(take_rows_gpu(qi.view(-1, 3 * D)[:, D:2 * D], ids), wk, "k in place")
    # guarded [L, 2D] output
    pad = 4096
    n = w.rows * 2 * D
    buf = torch.full((n + 2 * pad,), 1.5, dtype=qkv.dtype, device=DEV)
    o = buf[pad:pad + n].view(w.B, w.L, 2 * D)
    api.qknorm_rope3d(qkv, *args, q_out=o[..., :D], k_out=o[..., D:], **kw)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == 1.5) and torch.all(buf[-pad:] == 1.5)
    assert_close(take_rows_gpu(o.view(-1, 2 * D)[:, :D], ids), wq, "q guarded")


@ROPE
def test_qknorm_rope3d_large_positions_are_accurate(tab):
    # audio positions up to 4679 (15 s clip): angles reach thousands of radians
    B, T, H, W, na, nh, hd = 1, 0, 0, 0, 4680, 4, 128
    L = na
    qkv = activation(L, 3 * nh * hd, torch.bfloat16, DEV, 77, outliers=False).view(1, L, -1)
    q, k = api.qknorm_rope3d(qkv, T, H, W, na, nh, hd, table=_table(tab, T, H, W, na, hd))
    ids = np.arange(L - 300, L)
    wq, wk = oracle.qknorm_rope3d(take_rows(qkv.view(L, -1), ids), T, H, W, na, nh, hd,
                                  (16, 24, 24), 1e-6, 1e4, row_ids=ids)
    assert_close(take_rows_gpu(q.reshape(L, -1), ids), wq, "q far positions")
    assert_close(take_rows_gpu(k.reshape(L, -1), ids), wk, "k far positions")



# ----------------------------------------------------------------------------
# QKNorm + RoPE epilogue variants: layouts, half-split pairs, INT8 output
# ----------------------------------------------------------------------------

def _bshd(t, layout):
    """[B, L, H, hd] view of a q/k output in either layout."""
    return t if layout == "bshd" else t.permute(0, 2, 1, 3)


def _check_int8(codes, scales, want, n_heads, hd, what):
    """scale = max|x| / 127 per (row, head) within fp32 error, and every code
    dequantises to within half a step of the oracle value (plus 1% of a step
    for the fp32 arithmetic before the rounding)."""
    c = codes.detach().cpu().numpy().astype(np.float64).reshape(-1, n_heads, hd)
    sc = scales.detach().cpu().numpy().astype(np.float64).reshape(-1, n_heads)
    x = want.reshape(-1, n_heads, hd)
    np.testing.assert_allclose(sc, np.abs(x).max(axis=2) / 127.0, rtol=1e-5, atol=1e-12,
                               err_msg=f"{what} scales")
    err = np.abs(c * sc[:, :, None] - x)
    bound = sc[:, :, None] * 0.51 + 1e-9
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} codes off by more than half a step"
    assert np.abs(c).max() <= 127


@pytest.mark.parametrize("name", ("medium", "clip5s"))
@pytest.mark.parametrize("half", [False, True])
@pytest.mark.parametrize("layout", ["bshd", "bhsd"])
@pytest.mark.parametrize("int8", [False, True])
@ROPE
def test_qknorm_rope3d_ex_workload(name, half, layout, int8, tab):
    w = WORKLOADS[name]
    t = make_inputs(w, DEV, which=("qknorm_rope3d",))
    qkv = t["qkv"].view(w.B, w.L, 3 * w.D)
    res = api.qknorm_rope3d_ex(qkv, w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim,
                               w.sections, t["gamma_q"], t["gamma_k"], w.eps, w.theta,
                               layout=layout, half_split=half, int8=int8,
                               table=_table(tab, w.T, w.H, w.W, w.n_audio, w.head_dim))
    torch.cuda.synchronize()
    q, k = (_bshd(r, layout).reshape(w.rows, w.D) for r in res[:2])
    ids = None if name == "medium" else _ids(w, 512)
    qkv2 = qkv.view(-1, 3 * w.D)
    src = _o(qkv2) if ids is None else take_rows(qkv2[:, :2 * w.D], ids)
    wq, wk = oracle.qknorm_rope3d_ex(src, w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim,
                                     w.sections, w.eps, w.theta, half, _o(t["gamma_q"]),
                                     _o(t["gamma_k"]), row_ids=ids)
    if ids is not None:
        q, k = take_rows_gpu(q, ids), take_rows_gpu(k, ids)
    tag = f"ex[{name} half={half} {layout} int8={int8} table={tab}]"
    if int8:
        qs, ks = (r.reshape(w.rows, w.n_heads) for r in res[2:])
        if ids is not None:
            qs, ks = take_rows_gpu(qs, ids), take_rows_gpu(ks, ids)
        _check_int8(q, qs, wq, w.n_heads, w.head_dim, tag + " q")
        _check_int8(k, ks, wk, w.n_heads, w.head_dim, tag + " k")
    else:
        assert_close(q, wq, tag + " q")
        assert_close(k, wk, tag + " k")


@pytest.mark.parametrize("name", ("medium", "clip5s"))
@pytest.mark.parametrize("half", [False, True])
@pytest.mark.parametrize("int8", [False, True])
@ROPE
def test_qknorm_rope3d_ex_per_axis_freq(name, half, int8, tab):
    # each rotary section with a frequency ladder of its own, theta^(-j/s)
    w = WORKLOADS[name]
    t = make_inputs(w, DEV, which=("qknorm_rope3d",))
    qkv = t["qkv"].view(w.B, w.L, 3 * w.D)
    res = api.qknorm_rope3d_ex(qkv, w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim,
                               w.sections, t["gamma_q"], t["gamma_k"], w.eps, w.theta,
                               layout="bhsd", half_split=half, int8=int8, per_axis_freq=True,
                               table=_table(tab, w.T, w.H, w.W, w.n_audio, w.head_dim,
                                            per_axis=True))
    torch.cuda.synchronize()
    q, k = (_bshd(r, "bhsd").reshape(w.rows, w.D) for r in res[:2])
    ids = None if name == "medium" else _ids(w, 384)
    qkv2 = qkv.view(-1, 3 * w.D)
    src = _o(qkv2) if ids is None else take_rows(qkv2[:, :2 * w.D], ids)
    wq, wk = oracle.qknorm_rope3d_ex(src, w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim,
                                     w.sections, w.eps, w.theta, half, _o(t["gamma_q"]),
                                     _o(t["gamma_k"]), row_ids=ids, per_axis=True)
    if ids is not None:
        q, k = take_rows_gpu(q, ids), take_rows_gpu(k, ids)
    tag = f"per-axis[{name} half={half} int8={int8} table={tab}]"
    if int8:
        qs, ks = (r.reshape(w.rows, w.n_heads) for r in res[2:4])
        if ids is not None:
            qs, ks = take_rows_gpu(qs, ids), take_rows_gpu(ks, ids)
        _check_int8(q, qs, wq, w.n_heads, w.head_dim, tag + " q")
        _check_int8(k, ks, wk, w.n_heads, w.head_dim, tag + " k")
    else:
        assert_close(q, wq, tag + " q")
        assert_close(k, wk, tag + " k")


@pytest.mark.parametrize("name", ("medium", "clip5s"))
@pytest.mark.parametrize("layout", ["bshd", "bhsd"])
def test_qknorm_rope3d_ex_quantized_v(name, layout):
    # v quantised as it stands, per (row, head), next to the INT8 q and k
    w = WORKLOADS[name]
    t = make_inputs(w, DEV, which=("qknorm_rope3d",))
    qkv = t["qkv"].view(w.B, w.L, 3 * w.D)
    q, k, qs, ks, v, vs = api.qknorm_rope3d_ex(
        qkv, w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim, w.sections, t["gamma_q"],
        t["gamma_k"], w.eps, w.theta, layout=layout, int8=True, quantize_v=True)
    torch.cuda.synchronize()
    ids = None if name == "medium" else _ids(w, 384)
    qkv2 = qkv.view(-1, 3 * w.D)
    v_rows = qkv2[:, 2 * w.D:]
    want_v = oracle.widen(_o(v_rows.contiguous()) if ids is None else take_rows(v_rows, ids))
    v = _bshd(v, layout).reshape(w.rows, w.D)
    vs = vs.reshape(w.rows, w.n_heads)
    if ids is not None:
        v, vs = take_rows_gpu(v, ids), take_rows_gpu(vs, ids)
    _check_int8(v, vs, want_v, w.n_heads, w.head_dim, f"v[{name} {layout}]")
    # q and k are those of the INT8 entry point without v
    q2, k2, qs2, ks2 = api.qknorm_rope3d_ex(
        qkv, w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim, w.sections, t["gamma_q"],
        t["gamma_k"], w.eps, w.theta, layout=layout, int8=True)
    assert torch.equal(q, q2) and torch.equal(k, k2)
    assert torch.equal(qs, qs2) and torch.equal(ks, ks2)


@pytest.mark.parametrize("secs", [(64, 0, 0), (0, 32, 32), (20, 0, 44), (16, 24, 24),
                                  (18, 22, 24)])
@ROPE
def test_qknorm_rope3d_ex_per_axis_sections(secs, tab):
    # per-axis ladders with empty and uneven sections (an empty section holds
    # no pair, so its size never divides)
    B, T, H, W, na, nh, hd = 1, 4, 6, 5, 9, 4, 128
    L = T * H * W + na
    D = nh * hd
    qkv = activation(B * L, 3 * D, torch.bfloat16, DEV, 81, outliers=True).view(B, L, 3 * D)
    gq = vectors((hd,), 1.0, 0.1, torch.bfloat16, DEV, 82)
    gk = vectors((hd,), 1.0, 0.1, torch.bfloat16, DEV, 83)
    table = _table(tab, T, H, W, na, hd, secs, per_axis=True)
    for half in (False, True):
        wq, wk = oracle.qknorm_rope3d_ex(_o(qkv.view(B * L, 3 * D)), T, H, W, na, nh, hd, secs,
                                         1e-6, 1e4, half, _o(gq), _o(gk), per_axis=True)
        q, k = api.qknorm_rope3d_ex(qkv, T, H, W, na, nh, hd, secs, gq, gk, half_split=half,
                                    per_axis_freq=True, table=table)
        assert_close(q.reshape(B * L, D), wq, f"per-axis sections {secs} half={half} q")
        assert_close(k.reshape(B * L, D), wk, f"per-axis sections {secs} half={half} k")
        # INT8 too: a section edge inside a lane's 4 pairs (18, 22, 24) takes
        # the table rows' 4-byte copies
        q8, k8, qs, ks = api.qknorm_rope3d_ex(qkv, T, H, W, na, nh, hd, secs, gq, gk,
                                              half_split=half, per_axis_freq=True, int8=True,
                                              table=table)
        torch.cuda.synchronize()
        tag = f"per-axis sections {secs} half={half} int8"
        _check_int8(q8.reshape(B * L, D), qs, wq, nh, hd, tag + " q")
        _check_int8(k8.reshape(B * L, D), ks, wk, nh, hd, tag + " k")


def test_qknorm_rope3d_packed_qk_input():
    # a [B, L, 2D] tensor holding only q and k (ld_qkv = 2D, the form the
    # end-to-end path copies to the device) gives the same q and k, bit for
    # bit, as the merged [B, L, 3D] rows
    w = WORKLOADS["medium"]
    t = make_inputs(w, DEV, which=("qknorm_rope3d",))
    qkv = t["qkv"].view(w.B, w.L, 3 * w.D)
    packed = qkv[..., :2 * w.D].contiguous()
    args = (w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim, w.sections, t["gamma_q"],
            t["gamma_k"], w.eps, w.theta)
    q0, k0 = api.qknorm_rope3d(qkv, *args)
    q1, k1 = api.qknorm_rope3d(packed, *args)
    assert torch.equal(q0, q1) and torch.equal(k0, k1)
    for kw in ({"layout": "bhsd"}, {"int8": True}):
        r0 = api.qknorm_rope3d_ex(qkv, *args, **kw)
        r1 = api.qknorm_rope3d_ex(packed, *args, **kw)
        assert all(torch.equal(a, b) for a, b in zip(r0, r1))


@ROPE
def test_qknorm_rope3d_ex_interleaved_matches_default_entry_point(tab):
    # same arithmetic as sol_qknorm_rope3d (sol_qknorm_rope3d_tab), only the
    # addressing differs: bit-identical results in both layouts
    w = WORKLOADS["medium"]
    t = make_inputs(w, DEV, which=("qknorm_rope3d",))
    qkv = t["qkv"].view(w.B, w.L, 3 * w.D)
    args = (w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim, w.sections, t["gamma_q"],
            t["gamma_k"], w.eps, w.theta)
    table = _table(tab, w.T, w.H, w.W, w.n_audio, w.head_dim)
    q0, k0 = api.qknorm_rope3d(qkv, *args, table=table)
    for layout in ("bshd", "bhsd"):
        q1, k1 = api.qknorm_rope3d_ex(qkv, *args, layout=layout, table=table)
        assert torch.equal(_bshd(q1, layout).reshape(q0.shape), q0)
        assert torch.equal(_bshd(k1, layout).reshape(k0.shape), k0)


INT8_CASES = [c for c in QK_CASES if c[6] >= 64 and c[8] == torch.bfloat16]


@pytest.mark.parametrize("B,T,H,W,na,nh,hd,secs,dt,pad", INT8_CASES)
@ROPE
def test_qknorm_rope3d_ex_int8_cases(B, T, H, W, na, nh, hd, secs, dt, pad, tab):
    # the interleaved INT8 kernel on the QK edge shapes: audio only, video
    # only, one row, a ragged lane tail (41 heads), the widest row, padded
    # rows, and CTA shares (q and k CTAs of a pair) that cross W, H, the
    # video/audio split and samples
    L = T * H * W + na
    D = nh * hd
    C = 3 * D + pad
    qkv = activation(B * L, C, dt, DEV, 91, outliers=True).view(B, L, C)
    gq = vectors((hd,), 1.0, 0.1, dt, DEV, 92)
    gk = vectors((hd,), 1.0, 0.1, dt, DEV, 93)
    q, k, qs, ks = api.qknorm_rope3d_ex(qkv, T, H, W, na, nh, hd, secs, gq, gk, int8=True,
                                        table=_table(tab, T, H, W, na, hd, secs))
    torch.cuda.synchronize()
    wq, wk = oracle.qknorm_rope3d_ex(_o(qkv.view(B * L, C)), T, H, W, na, nh, hd, secs,
                                     1e-6, 1e4, False, _o(gq), _o(gk))
    tag = f"int8 B={B} T={T} H={H} W={W} na={na} nh={nh} hd={hd} table={tab}"
    _check_int8(q.reshape(B * L, D), qs, wq, nh, hd, tag + " q")
    _check_int8(k.reshape(B * L, D), ks, wk, nh, hd, tag + " k")


@pytest.mark.parametrize("hd,secs", [(64, (8, 12, 12)), (256, (32, 48, 48))])
@pytest.mark.parametrize("half", [False, True])
@pytest.mark.parametrize("per_axis", [False, True])
@ROPE
def test_qknorm_rope3d_ex_head_dims(hd, secs, half, per_axis, tab):
    B, T, H, W, na, nh = 2, 3, 5, 7, 11, 6
    L = T * H * W + na
    D = nh * hd
    qkv = activation(B * L, 3 * D, torch.bfloat16, DEV, 61, outliers=True).view(B, L, 3 * D)
    gq = vectors((hd,), 1.0, 0.1, torch.bfloat16, DEV, 62)
    gk = vectors((hd,), 1.0, 0.1, torch.bfloat16, DEV, 63)
    wq, wk = oracle.qknorm_rope3d_ex(_o(qkv.view(B * L, 3 * D)), T, H, W, na, nh, hd, secs,
                                     1e-6, 1e4, half, _o(gq), _o(gk), per_axis=per_axis)
    tag = f"hd={hd} half={half} per_axis={per_axis} table={tab}"
    table = _table(tab, T, H, W, na, hd, secs, per_axis=per_axis)
    for int8 in (False, True):
        res = api.qknorm_rope3d_ex(qkv, T, H, W, na, nh, hd, secs, gq, gk, layout="bhsd",
                                   half_split=half, int8=int8, per_axis_freq=per_axis,
                                   quantize_v=int8, table=table)
        q, k = (_bshd(r, "bhsd").reshape(B * L, D) for r in res[:2])
        if int8:
            _check_int8(q, res[2], wq, nh, hd, tag + " q")
            _check_int8(k, res[3], wk, nh, hd, tag + " k")
            # v, quantised as it stands (G = hd/8 lanes per head in its kernel too)
            want_v = oracle.widen(_o(qkv.view(B * L, 3 * D)[:, 2 * D:].contiguous()))
            _check_int8(_bshd(res[4], "bhsd").reshape(B * L, D), res[5], want_v, nh, hd,
                        tag + " v")
        else:
            assert_close(q, wq, tag + " q")
            assert_close(k, wk, tag + " k")



# ----------------------------------------------------------------------------
# GEMM + bias + GELU (tcgen05)
# ----------------------------------------------------------------------------

def _weights(N, K, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return (torch.randn((N, K), generator=g, device=DEV) / K ** 0.5).to(torch.bfloat16)


GEMM_SHAPES = [
    (1, 8, 8), (127, 256, 64), (300, 520, 1032), (257, 384, 256), (1000, 1024, 5120),
    (129, 264, 72),
]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_gelu_shapes(M, N, K):
    A = activation(M, K, torch.bfloat16, DEV, 101 + M, outliers=True)
    Bw = _weights(N, K, 102 + N)
    bias = vectors((N,), 0.0, 0.5, torch.bfloat16, DEV, 103)
    for b in (None, bias):
        C = api.gemm_gelu(A, Bw, b)
        want = oracle.gemm_gelu(_o(A), _o(Bw), None if b is None else _o(b))
        assert_close(C, want, f"gemm_gelu M={M} N={N} K={K} bias={b is not None}")


def test_gemm_gelu_clip_mlp_shape_sampled():
    # the 5 s clip's MLP up-projection: 126,552 tokens x (5120 -> 4 x 5120)
    w = WORKLOADS["clip5s"]
    M, K, N = w.rows, w.D, 4 * w.D
    A = activation(M, K, torch.bfloat16, DEV, 104, outliers=True)
    Bw = _weights(N, K, 105)
    bias = vectors((N,), 0.0, 0.5, torch.bfloat16, DEV, 106)
    C = api.gemm_gelu(A, Bw, bias)
    torch.cuda.synchronize()
    ids = sample_rows(M, w.L, w.n_video, w.B, 192, seed=107)
    want = oracle.gemm_gelu(take_rows(A, ids), _o(Bw), _o(bias))
    assert_close(take_rows_gpu(C, ids), want, "gemm_gelu clip MLP sampled")
    C2 = api.gemm_gelu(A[:4096], Bw, bias)
    assert torch.equal(C2, C[:4096])  # same tiles, same order: deterministic


@pytest.mark.parametrize("half", [False, True])
@ROPE
def test_qknorm_rope3d_ex_int8_edge_heads(half, tab):
    # per row: a normal head, an all-zero head, a head of tiny normal values
    # (x * 2^-110, so max|u| < 2^-96 and the kernel rescales before dividing),
    # and a head with one 1e4 outlier; q, k and v get different heads
    T, H, W, na, nh, hd = 2, 3, 4, 5, 4, 128
    L = T * H * W + na
    D = nh * hd
    base = activation(L, 3 * D, torch.float32, DEV, 71, outliers=False).view(L, 3, nh, hd)
    x = base.clone()
    for part, (zero, tiny, spike) in enumerate([(1, 2, 3), (2, 3, 1), (3, 1, 2)]):
        x[:, part, zero] = 0.0
        x[:, part, tiny] = torch.sign(base[:, part, tiny]) * (1 + base[:, part, tiny].abs()) * 2.0 ** -110
        x[:, part, spike, 17] = 1.0e4
    qkv = x.to(torch.bfloat16).view(1, L, 3 * D)
    gq = vectors((hd,), 1.0, 0.1, torch.bfloat16, DEV, 72)
    gk = vectors((hd,), 1.0, 0.1, torch.bfloat16, DEV, 73)
    res = api.qknorm_rope3d_ex(qkv, T, H, W, na, nh, hd, (16, 24, 24), gq, gk, layout="bshd",
                               half_split=half, int8=True, quantize_v=True,
                               table=_table(tab, T, H, W, na, hd))
    torch.cuda.synchronize()
    wq, wk = oracle.qknorm_rope3d_ex(_o(qkv.view(L, 3 * D)), T, H, W, na, nh, hd, (16, 24, 24),
                                     1e-6, 1e4, half, _o(gq), _o(gk))
    q, k, qs, ks, v, vs = res
    want_v = oracle.widen(_o(qkv.view(L, 3 * D)[:, 2 * D:].contiguous()))
    _check_int8(v.reshape(L, D), vs, want_v, nh, hd, f"edge half={half} v")
    assert torch.all(vs.view(L, nh)[:, 3] == 0) and torch.all(v.view(L, nh, hd)[:, 3] == 0)
    assert int(v.view(L, nh, hd)[:, 1].abs().amax()) == 127
    _check_int8(q.reshape(L, D), qs, wq, nh, hd, f"edge half={half} q")
    _check_int8(k.reshape(L, D), ks, wk, nh, hd, f"edge half={half} k")
    # the zero heads: scale 0 and every code 0
    assert torch.all(qs.view(L, nh)[:, 1] == 0) and torch.all(q.view(L, nh, hd)[:, 1] == 0)
    assert torch.all(ks.view(L, nh)[:, 2] == 0) and torch.all(k.view(L, nh, hd)[:, 2] == 0)
    # the tiny heads use the full code range
    assert int(q.view(L, nh, hd)[:, 2].abs().amax()) == 127


# ----------------------------------------------------------------------------
# Rotary table (sol_rope_table_build) and the table-driven entry points
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("hd,secs,per_axis", [(128, (16, 24, 24), False),
                                              (128, (16, 24, 24), True),
                                              (64, (8, 12, 12), True), (16, (2, 3, 3), False)])
def test_rope_table_entries(hd, secs, per_axis):
    # row p: cos(p f_i) for every pair i, then sin(p f_i); each entry the fp64
    # value rounded once to fp32 (within half an fp32 ulp, plus the fp64
    # sincos error)
    n_pos = 4680
    tab = api.RopeTable(n_pos, hd, secs, 1e4, per_axis, device=DEV)
    got = tab.data.view(n_pos, hd).double().cpu().numpy()
    npairs = hd // 2
    i = np.arange(npairs)
    if per_axis:
        start = np.concatenate([np.full(s, sum(secs[:a])) for a, s in enumerate(secs)])
        size = np.concatenate([np.full(s, s) for s in secs])
        f = 1e4 ** (-(i - start) / size)
    else:
        f = 1e4 ** (-2.0 * i / hd)
    ang = np.arange(n_pos, dtype=np.float64)[:, None] * f[None, :]
    want = np.concatenate([np.cos(ang), np.sin(ang)], axis=1)
    err = np.abs(got - want)
    assert err.max() <= 2.0 ** -24 * 1.01 + 1e-15, err.max()


def test_rope_table_zero_positions_and_reuse():
    # n_pos = 0 is a no-op build; a table is reused across calls and samples
    tab0 = api.RopeTable(0, 128, device=DEV)
    assert tab0.n_pos == 0
    w = WORKLOADS["medium"]
    t = make_inputs(w, DEV, which=("qknorm_rope3d",))
    qkv = t["qkv"].view(w.B, w.L, 3 * w.D)
    table = _table(True, w.T, w.H, w.W, w.n_audio, w.head_dim)
    args = (w.T, w.H, w.W, w.n_audio, w.n_heads, w.head_dim, w.sections, t["gamma_q"],
            t["gamma_k"], w.eps, w.theta)
    q0, k0 = api.qknorm_rope3d(qkv, *args, table=table)
    q1, k1 = api.qknorm_rope3d(qkv, *args, table=table)
    assert torch.equal(q0, q1) and torch.equal(k0, k1)
    # the table path differs from the on-the-fly one only by the rounding of
    # (cos, sin): at most a bf16 ulp or two of the output, on few elements
    q2, _ = api.qknorm_rope3d(qkv, *args)
    d = (q2.float() - q0.float()).abs()
    assert float(d.max()) <= 2.0 ** -6 * float(q0.float().abs().max())
    assert float((d > 0).float().mean()) < 0.05


def test_rope_table_too_small_or_overlapping_is_rejected():
    # the host refuses a table with too few positions, or an output over the
    # table, before launching anything
    T, H, W, na, nh, hd = 2, 3, 4, 5, 2, 128
    L = T * H * W + na
    D = nh * hd
    qkv = activation(L, 3 * D, torch.bfloat16, DEV, 91, outliers=False).view(1, L, 3 * D)
    small = api.RopeTable(4, hd, device=DEV)   # needs max(T, H, W, na) = 5
    with pytest.raises(_abi.SolError, match="positions"):
        api.qknorm_rope3d(qkv, T, H, W, na, nh, hd, table=small)
    ok = api.RopeTable(5, hd, device=DEV)
    api.qknorm_rope3d(qkv, T, H, W, na, nh, hd, table=ok)
    # an output that overlaps the table
    big = api.RopeTable(2 * L * D // hd + 8, hd, device=DEV)
    before = big.data.clone()
    out = big.data.view(torch.bfloat16)[:L * 2 * D].view(1, L, 2 * D)
    with pytest.raises(_abi.SolError, match="table"):
        api.qknorm_rope3d(qkv, T, H, W, na, nh, hd, table=big, q_out=out[..., :D],
                          k_out=out[..., D:])
    torch.cuda.synchronize()
    assert torch.equal(big.data, before)
    # per-axis flag of the layout and the table must agree
    pa = api.RopeTable(5, hd, per_axis_freq=True, device=DEV)
    with pytest.raises(ValueError):
        api.qknorm_rope3d_ex(qkv, T, H, W, na, nh, hd, table=pa)


# ----------------------------------------------------------------------------
# Row order: the chunk of rows dealt to each CTA shrinks for small inputs
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("rows", [5000, 18945, 37887, 47361, 94721])
def test_row_order_regimes(rows):
    # The kernels deal rows to CTAs in chunks of up to 8 rows, halved while
    # the CTAs would get fewer than 16 chunks; row counts on both sides of the
    # B200's halving points (resident CTAs x chunk x 16) take different chunk
    # sizes.  Every row must come out once and right: sampled rows (with the
    # first, the last and the video/audio boundary) against the oracle, and
    # the whole output against the same rows in two calls, bit for bit (each
    # row's arithmetic does not depend on which CTA takes it).
    D, nv = 5120, rows - 97
    x = activation(rows, D, torch.bfloat16, DEV, 201, outliers=True)
    h = activation(rows, D, torch.bfloat16, DEV, 202, outliers=True)
    br = activation(rows, D, torch.bfloat16, DEV, 203, outliers=True)
    sc = vectors((1, 2, D), 0.0, 0.5, torch.bfloat16, DEV, 204)
    sh = vectors((1, 2, D), 0.0, 0.5, torch.bfloat16, DEV, 205)
    gt = vectors((1, 2, D), 0.0, 0.1, torch.bfloat16, DEV, 206)
    y = api.rms_adaln(x.view(1, rows, D), sc, sh, nv)
    out = api.gate_residual(h.view(1, rows, D), br.view(1, rows, D), gt, nv)
    torch.cuda.synchronize()
    ids = sample_rows(rows, rows, nv, 1, 256, seed=207)
    ids = np.unique(np.concatenate([ids, [0, rows - 1, nv - 1, nv]]))
    assert_close(take_rows_gpu(y.view(rows, D), ids),
                 oracle.rms_adaln(take_rows(x, ids), _o(sc), _o(sh), rows, nv, 1e-6,
                                  row_ids=ids), f"rms rows={rows}")
    assert_close(take_rows_gpu(out.view(rows, D), ids),
                 oracle.gate_residual(take_rows(h, ids), take_rows(br, ids), _o(gt), rows, nv,
                                      row_ids=ids), f"gate rows={rows}")
    # the same rows in two calls (other row counts, so other chunk sizes and
    # other CTAs per row): bit-identical to the one call
    k = rows // 3
    y2 = torch.cat([api.rms_adaln(x[:k].view(1, k, D), sc, sh, k),
                    api.rms_adaln(x[k:].view(1, rows - k, D), sc, sh, nv - k)], dim=1)
    o2 = torch.cat([api.gate_residual(h[:k].view(1, k, D), br[:k].view(1, k, D), gt, k),
                    api.gate_residual(h[k:].view(1, rows - k, D), br[k:].view(1, rows - k, D),
                                      gt, nv - k)], dim=1)
    torch.cuda.synchronize()
    assert torch.equal(y2, y)
    assert torch.equal(o2, out)


def test_rms_adaln_guarded_and_unguarded_agree():
    # At D = 5120 the 128 x 5 split covers a row exactly; launches of up to
    # 16,384 rows take the kernel without per-slot bounds checks, longer ones
    # the guarded kernel.  16,385 rows (guarded) and their first 16,384 rows
    # alone (unguarded) must give the same bits on those rows, and both
    # must match the oracle on sampled rows.
    D, rows = 5120, 16385
    nv = rows - 201
    x = activation(rows, D, torch.bfloat16, DEV, 211, outliers=True)
    sc = vectors((1, 2, D), 0.0, 0.5, torch.bfloat16, DEV, 212)
    sh = vectors((1, 2, D), 0.0, 0.5, torch.bfloat16, DEV, 213)
    y_long = api.rms_adaln(x.view(1, rows, D), sc, sh, nv)
    y_short = api.rms_adaln(x[:rows - 1].view(1, rows - 1, D), sc, sh, nv)
    torch.cuda.synchronize()
    assert torch.equal(y_short.view(rows - 1, D), y_long.view(rows, D)[:rows - 1])
    ids = sample_rows(rows, rows, nv, 1, 256, seed=214)
    ids = np.unique(np.concatenate([ids, [0, rows - 1, nv - 1, nv]]))
    assert_close(take_rows_gpu(y_long.view(rows, D), ids),
                 oracle.rms_adaln(take_rows(x, ids), _o(sc), _o(sh), rows, nv, 1e-6,
                                  row_ids=ids), "rms guarded")
