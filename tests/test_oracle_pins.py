"""Pins for the fp64 CPU oracle, independent of the oracle's own code.

Each test checks the oracle against something the definitions or the
workload text fix by themselves: hand-worked values (tests/golden), closed
forms, invariants of RMSNorm and of rotations, textbook special cases
(complex multiplication, an explicit block-diagonal rotation matrix) and
brute force on tiny inputs.  Together they are meant to fail on any
plausible slip in the oracle: eps outside the root, a mean over D-1, a
missing "1 +", swapped scale/shift, a wrong modality or sample index,
normalising over D instead of per head, swapped gamma_q/gamma_k, reading v,
a wrong rotation sign, the half-split pair layout, per-axis restarted
frequencies, a wrong axis or position mapping, wrong audio positions.
"""
import math

import numpy as np
import pytest

import oracle
from tests.conftest import read_golden

RNG = np.random.default_rng(12345)


def f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def bf16_bits(a):
    """Exact bf16 bits of float32 values that bf16 represents exactly."""
    a = f32(a)
    bits = a.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0), "value not exactly representable in bf16"
    return (bits >> 16).astype(np.uint16)


# ----------------------------------------------------------------------------
# RMS-AdaLN
# ----------------------------------------------------------------------------

def _hand():
    g = read_golden("rms_adaln_hand.txt")
    return {k: np.array(v[0], dtype=np.float64) for k, v in g.items()}


def _hand_inputs(conv):
    h = _hand()
    x = conv(np.stack([h["x0"], h["x1"]]))
    scale = conv(np.stack([h["scale_video"], h["scale_audio"]])[None])
    shift = conv(np.stack([h["shift_video"], h["shift_audio"]])[None])
    return h, x, scale, shift, conv(h["gamma"])


@pytest.mark.parametrize("conv", [f32, bf16_bits], ids=["f32", "bf16"])
def test_rms_adaln_hand_worked(conv):
    h, x, scale, shift, gamma = _hand_inputs(conv)
    y = oracle.rms_adaln(x, scale, shift, L=2, n_video=1, eps=0.0)
    np.testing.assert_allclose(y[0], h["y0"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(y[1], h["y1"], rtol=0, atol=1e-14)
    yg = oracle.rms_adaln(x, scale, shift, L=2, n_video=1, eps=0.0, gamma=gamma)
    np.testing.assert_allclose(yg[0], h["y0_gamma"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(yg[1], h["y1_gamma"], rtol=0, atol=1e-14)


@pytest.mark.parametrize("c,eps,expect", [(1.0, 3.0, 0.5), (2.0, 5.0, 2.0 / 3.0),
                                          (-4.0, 9.0, -0.8)])
def test_rms_adaln_constant_row_closed_form(c, eps, expect):
    # x = c * ones(D), scale = shift = 0: y = c / sqrt(c^2 + eps) in every channel
    D = 64
    x = f32(np.full((1, D), c))
    z = f32(np.zeros((1, 2, D)))
    y = oracle.rms_adaln(x, z, z, L=1, n_video=1, eps=eps)
    np.testing.assert_allclose(y, expect, rtol=1e-15, atol=0)


def test_rms_adaln_unit_rms():
    D, rows, eps = 96, 7, 1e-6
    x = f32(RNG.standard_normal((rows, D)) * np.linspace(0.01, 30, rows)[:, None])
    z = f32(np.zeros((1, 2, D)))
    y = oracle.rms_adaln(x, z, z, L=rows, n_video=3, eps=eps)
    ms = np.mean(x.astype(np.float64) ** 2, axis=1)
    np.testing.assert_allclose(np.sqrt(np.mean(y ** 2, axis=1)),
                               np.sqrt(ms / (ms + eps)), rtol=1e-13)


def test_rms_adaln_modality_and_sample_select():
    # scale = -1 makes y = shift exactly; shift[b, m] = 10*b + m + 1 marks the
    # (sample, modality) each row must pick: rows r < n_video are video.
    B, L, n_video, D = 2, 5, 3, 8
    x = f32(RNG.standard_normal((B * L, D)))
    scale = f32(np.full((B, 2, D), -1.0))
    shift = f32(np.array([[[10 * b + m + 1] * D for m in range(2)] for b in range(B)]))
    y = oracle.rms_adaln(x, scale, shift, L=L, n_video=n_video, eps=1e-6)
    for g in range(B * L):
        b, r = divmod(g, L)
        m = 0 if r < n_video else 1
        assert np.all(y[g] == 10 * b + m + 1), (g, y[g])


def test_rms_adaln_positive_scale_invariance():
    D = 40
    x = f32(RNG.standard_normal((3, D)))
    sc = f32(RNG.standard_normal((1, 2, D)))
    sh = f32(RNG.standard_normal((1, 2, D)))
    y1 = oracle.rms_adaln(x, sc, sh, L=3, n_video=2, eps=0.0)
    y2 = oracle.rms_adaln(f32(x * 8.0), sc, sh, L=3, n_video=2, eps=0.0)
    np.testing.assert_allclose(y1, y2, rtol=1e-13, atol=1e-13)


def test_rms_adaln_affine_in_modulation():
    # y is affine in (scale, shift): y(2a, 2b) - y(a, b) == y(a, b) - y(0, 0)
    D = 24
    x = f32(RNG.standard_normal((2, D)))
    a = RNG.standard_normal((1, 2, D)).astype(np.float32)
    b = RNG.standard_normal((1, 2, D)).astype(np.float32)
    z = f32(np.zeros_like(a))
    y0 = oracle.rms_adaln(x, z, z, L=2, n_video=1, eps=1e-6)
    y1 = oracle.rms_adaln(x, f32(a), f32(b), L=2, n_video=1, eps=1e-6)
    y2 = oracle.rms_adaln(x, f32(2 * a), f32(2 * b), L=2, n_video=1, eps=1e-6)
    np.testing.assert_allclose(y2 - y1, y1 - y0, rtol=1e-12, atol=1e-12)


def test_rms_adaln_bf16_widening_bits():
    # 0x3F80 = 1.0, 0xC000 = -2.0, 0x4049 = 3.140625 (bf16 patterns)
    D = 3
    x = np.array([[0x3F80, 0xC000, 0x4049]], dtype=np.uint16)
    z = np.zeros((1, 2, D), dtype=np.uint16)  # +0.0
    y = oracle.rms_adaln(x, z, z, L=1, n_video=1, eps=0.0)
    v = np.array([1.0, -2.0, 3.140625])
    np.testing.assert_allclose(y[0], v / math.sqrt(np.mean(v ** 2)), rtol=1e-15)


def test_rms_adaln_row_ids_pick_rows():
    B, L, n_video, D = 2, 6, 4, 16
    x = f32(RNG.standard_normal((B * L, D)))
    sc = f32(RNG.standard_normal((B, 2, D)))
    sh = f32(RNG.standard_normal((B, 2, D)))
    full = oracle.rms_adaln(x, sc, sh, L=L, n_video=n_video, eps=1e-6)
    ids = np.array([11, 0, 4, 3, 6], dtype=np.int64)
    part = oracle.rms_adaln(x[ids], sc, sh, L=L, n_video=n_video, eps=1e-6, row_ids=ids)
    np.testing.assert_array_equal(part, full[ids])


def test_rms_adaln_rejects_bad_sizes():
    x = f32(np.ones((2, 4)))
    z = f32(np.zeros((1, 2, 4)))
    with pytest.raises(ValueError):
        oracle.rms_adaln(x, z, z, L=2, n_video=3, eps=1e-6)


# ----------------------------------------------------------------------------
# Gated residual
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("conv", [f32, bf16_bits], ids=["f32", "bf16"])
def test_gate_residual_hand_worked(conv):
    h = _hand()
    hh = conv(h["h"][None])
    br = conv(h["branch"][None])
    gate = conv(np.stack([h["gate_video"], np.zeros(4)])[None])
    out = oracle.gate_residual(hh, br, gate, L=1, n_video=1)
    np.testing.assert_array_equal(out[0], h["out"])


def test_gate_residual_zero_and_one():
    B, L, D = 1, 5, 32
    hh = f32(RNG.standard_normal((L, D)))
    br = f32(RNG.standard_normal((L, D)))
    out0 = oracle.gate_residual(hh, br, f32(np.zeros((B, 2, D))), L=L, n_video=2)
    np.testing.assert_array_equal(out0, hh.astype(np.float64))
    out1 = oracle.gate_residual(hh, br, f32(np.ones((B, 2, D))), L=L, n_video=2)
    np.testing.assert_array_equal(out1, hh.astype(np.float64) + br.astype(np.float64))


def test_gate_residual_modality_and_sample_select():
    B, L, n_video, D = 2, 4, 1, 8
    hh = f32(np.zeros((B * L, D)))
    br = f32(np.ones((B * L, D)))
    gate = f32(np.array([[[10 * b + m + 1] * D for m in range(2)] for b in range(B)]))
    out = oracle.gate_residual(hh, br, gate, L=L, n_video=n_video)
    for g in range(B * L):
        b, r = divmod(g, L)
        assert np.all(out[g] == 10 * b + (0 if r < n_video else 1) + 1)


# ----------------------------------------------------------------------------
# QKNorm + 3D RoPE
# ----------------------------------------------------------------------------

TINY = dict(T=2, H=4, W=6, n_audio=8, n_heads=2, head_dim=128,
            sections=(16, 24, 24), theta=10000.0)


def _grid_rows(T, H, W, n_audio, **_):
    return T * H * W + n_audio


def _qkv_same_every_row(q_head, k_head, rows, n_heads, v_fill=0.0, pad=0, pad_fill=0.0):
    hd = q_head.shape[-1]
    D = n_heads * hd
    row = np.concatenate([np.tile(q_head, n_heads), np.tile(k_head, n_heads),
                          np.full(D, v_fill), np.full(pad, pad_fill)])
    return f32(np.tile(row, (rows, 1)))


def _positions():
    g = read_golden("rope3d_tiny_positions.txt")
    pos = {int(r[0]): (int(r[1]), int(r[2]), int(r[3])) for r in g["pos"]}
    pairs = {int(p[0]): ("thw".index(p[1]), float(p[2])) for p in g["pair"]}
    return pos, pairs


def _wrap(a):
    return (a + np.pi) % (2 * np.pi) - np.pi


def test_rope_angles_match_hand_table():
    # every pair of q holds (1, 0) and of k holds (0, 1): with eps = 0 and no
    # gamma the normalised pair is (sqrt2, 0) / (0, sqrt2); after rotation by
    # phi, q's pair is sqrt2 (cos phi, sin phi) and k's sqrt2 (-sin phi, cos phi).
    pos, pairs = _positions()
    rows = _grid_rows(**TINY)
    hd = TINY["head_dim"]
    qh = np.tile([1.0, 0.0], hd // 2)
    kh = np.tile([0.0, 1.0], hd // 2)
    qkv = _qkv_same_every_row(qh, kh, rows, TINY["n_heads"])
    q, k = oracle.qknorm_rope3d(qkv, eps=0.0, **TINY)
    s2 = math.sqrt(2.0)
    for r, p in pos.items():
        for i, (axis, freq) in pairs.items():
            phi = p[axis] * freq
            for head in range(TINY["n_heads"]):
                a, b = q[r, head * hd + 2 * i], q[r, head * hd + 2 * i + 1]
                assert abs(math.hypot(a, b) - s2) < 1e-13
                assert abs(_wrap(math.atan2(b, a) - phi)) < 1e-12, (r, i, head)
                c, d = k[r, head * hd + 2 * i], k[r, head * hd + 2 * i + 1]
                np.testing.assert_allclose([c, d], [-s2 * math.sin(phi), s2 * math.cos(phi)],
                                           atol=1e-13)


@pytest.mark.parametrize("half", [False, True])
def test_rope_per_axis_angles_match_hand_table(half):
    # per-axis ladder: every pair of q holds (1, 0) and of k holds (0, 1) in
    # the chosen pair layout; with eps = 0 the rotated q pair is
    # sqrt2 (cos phi, sin phi), phi = position on the pair's axis times the
    # hand-written per-axis frequency
    pos, _ = _positions()
    g = read_golden("rope3d_per_axis_freqs.txt")
    pairs = {int(r[0]): ("thw".index(r[1]), float(r[3])) for r in g["pair"]}
    rows = _grid_rows(**TINY)
    hd = TINY["head_dim"]
    if half:
        qh = np.concatenate([np.ones(hd // 2), np.zeros(hd // 2)])
        kh = np.concatenate([np.zeros(hd // 2), np.ones(hd // 2)])
    else:
        qh, kh = np.tile([1.0, 0.0], hd // 2), np.tile([0.0, 1.0], hd // 2)
    qkv = _qkv_same_every_row(qh, kh, rows, TINY["n_heads"])
    q, k = oracle.qknorm_rope3d_ex(qkv, TINY["T"], TINY["H"], TINY["W"], TINY["n_audio"],
                                   TINY["n_heads"], hd, TINY["sections"], 0.0, TINY["theta"],
                                   half, per_axis=True)
    s2 = math.sqrt(2.0)
    for r, p in pos.items():
        for i, (axis, freq) in pairs.items():
            phi = p[axis] * freq
            ia, ib = (i, i + hd // 2) if half else (2 * i, 2 * i + 1)
            for head in range(TINY["n_heads"]):
                a, b = q[r, head * hd + ia], q[r, head * hd + ib]
                assert abs(math.hypot(a, b) - s2) < 1e-13
                assert abs(_wrap(math.atan2(b, a) - phi)) < 1e-12, (r, i, head)
                c, d = k[r, head * hd + ia], k[r, head * hd + ib]
                np.testing.assert_allclose([c, d], [-s2 * math.sin(phi), s2 * math.cos(phi)],
                                           atol=1e-13)


def test_rope_per_axis_with_one_section_is_the_global_ladder():
    # a single section of all 64 pairs: its own ladder theta^(-j/64) is the
    # global theta^(-2i/128), so the per-axis flag changes nothing
    rows = _grid_rows(**TINY)
    qkv = f32(RNG.standard_normal((rows, 3 * 2 * 128)))
    for secs in ((64, 0, 0), (0, 64, 0), (0, 0, 64)):
        args = (qkv, TINY["T"], TINY["H"], TINY["W"], TINY["n_audio"], 2, 128, secs, 1e-6,
                1e4)
        for half in (False, True):
            q0, k0 = oracle.qknorm_rope3d_ex(*args, half, per_axis=False)
            q1, k1 = oracle.qknorm_rope3d_ex(*args, half, per_axis=True)
            np.testing.assert_allclose(q1, q0, rtol=0, atol=1e-15)
            np.testing.assert_allclose(k1, k0, rtol=0, atol=1e-15)
    # and with three sections it differs (pair 16 is the h section's first)
    args = (qkv, TINY["T"], TINY["H"], TINY["W"], TINY["n_audio"], 2, 128, (16, 24, 24), 1e-6,
            1e4)
    q0, _ = oracle.qknorm_rope3d_ex(*args, False, per_axis=False)
    q1, _ = oracle.qknorm_rope3d_ex(*args, False, per_axis=True)
    assert np.abs(q1 - q0).max() > 0.1


def test_qknorm_identity_at_origin_gives_gamma():
    # a constant head at position (0,0,0) normalises to all ones (eps = 0) and
    # the rotation is the identity, so the output is gamma itself.
    hd = 128
    gq = f32(1.0 + 0.1 * RNG.standard_normal(hd))
    gk = f32(1.0 + 0.1 * RNG.standard_normal(hd))
    qkv = _qkv_same_every_row(np.full(hd, -3.5), np.full(hd, 0.25), 1, 2)
    q, k = oracle.qknorm_rope3d(qkv, 1, 1, 1, 0, 2, hd, (16, 24, 24), 0.0, 1e4,
                                gamma_q=gq, gamma_k=gk)
    np.testing.assert_allclose(q[0], np.tile(-gq.astype(np.float64), 2), rtol=1e-15)
    np.testing.assert_allclose(k[0], np.tile(gk.astype(np.float64), 2), rtol=1e-15)


def test_qknorm_is_per_head_and_rms_one():
    rows = _grid_rows(**TINY)
    hd, nh = 128, 2
    D = nh * hd
    qkv = RNG.standard_normal((rows, 3 * D))
    qkv[:, hd:2 * hd] *= 100.0          # q head 1 is 100x larger
    qkv[:, D:D + hd] *= 0.01            # k head 0 is 100x smaller
    qkv = f32(qkv)
    eps = 1e-6
    q, k = oracle.qknorm_rope3d(qkv, eps=eps, **TINY)
    for part, out, off in ((0, q, 0), (1, k, D)):
        for head in range(nh):
            x = qkv[:, off + head * hd: off + (head + 1) * hd].astype(np.float64)
            ms = np.mean(x ** 2, axis=1)
            got = np.sqrt(np.mean(out[:, head * hd:(head + 1) * hd] ** 2, axis=1))
            np.testing.assert_allclose(got, np.sqrt(ms / (ms + eps)), rtol=1e-12)


def test_qknorm_gamma_q_and_gamma_k_not_swapped():
    rows = _grid_rows(**TINY)
    qkv = f32(RNG.standard_normal((rows, 3 * 256)))
    gq = f32(np.full(128, 2.0))
    gk = f32(np.full(128, 3.0))
    q, k = oracle.qknorm_rope3d(qkv, eps=0.0, gamma_q=gq, gamma_k=gk, **TINY)
    np.testing.assert_allclose(np.sqrt(np.mean(q ** 2, axis=1)), 2.0, rtol=1e-13)
    np.testing.assert_allclose(np.sqrt(np.mean(k ** 2, axis=1)), 3.0, rtol=1e-13)


def test_qknorm_reads_neither_v_nor_row_padding():
    rows = _grid_rows(**TINY)
    qh, kh = RNG.standard_normal(128), RNG.standard_normal(128)
    clean = _qkv_same_every_row(qh, kh, rows, 2, v_fill=0.0, pad=8, pad_fill=0.0)
    dirty = _qkv_same_every_row(qh, kh, rows, 2, v_fill=np.nan, pad=8, pad_fill=np.inf)
    q0, k0 = oracle.qknorm_rope3d(clean, eps=1e-6, **TINY)
    q1, k1 = oracle.qknorm_rope3d(dirty, eps=1e-6, **TINY)
    np.testing.assert_array_equal(q0, q1)
    np.testing.assert_array_equal(k0, k1)


def _closed_form_angles(r, T=2, H=4, W=6, hd=128, sections=(16, 24, 24)):
    """Angles of the 64 pairs of row r from the raster rule and 10^(-i/16)."""
    nv = T * H * W
    if r < nv:
        p = (r // (H * W), (r // W) % H, r % W)
    else:
        p = (r - nv, 0, 0)
    st, sh, _ = sections
    ang = np.empty(hd // 2)
    for i in range(hd // 2):
        axis = 0 if i < st else (1 if i < st + sh else 2)
        ang[i] = p[axis] * 10.0 ** (-i / 16.0)
    return ang


def test_rope_is_complex_multiplication():
    # same random head at every row; row 0 sits at the origin (identity), so
    # row r must equal row 0 times exp(i * phi_r) pair by pair (numpy complex).
    rows = _grid_rows(**TINY)
    qh, kh = RNG.standard_normal(128), RNG.standard_normal(128)
    qkv = _qkv_same_every_row(qh, kh, rows, 2)
    q, k = oracle.qknorm_rope3d(qkv, eps=1e-6, **TINY)
    for out in (q, k):
        z0 = out[0, 0:128:2] + 1j * out[0, 1:128:2]
        for r in range(rows):
            rot = z0 * np.exp(1j * _closed_form_angles(r))
            for head in range(2):
                got = out[r, head * 128:(head + 1) * 128]
                np.testing.assert_allclose(got[0::2], rot.real, atol=1e-12)
                np.testing.assert_allclose(got[1::2], rot.imag, atol=1e-12)


def test_rope_equals_block_diagonal_rotation_matrix():
    rows = _grid_rows(**TINY)
    qh, kh = RNG.standard_normal(128), RNG.standard_normal(128)
    qkv = _qkv_same_every_row(qh, kh, rows, 2)
    q, _ = oracle.qknorm_rope3d(qkv, eps=1e-6, **TINY)
    for r in (1, 7, 31, 47, 55):
        R = np.zeros((128, 128))
        for i, a in enumerate(_closed_form_angles(r)):
            R[2 * i:2 * i + 2, 2 * i:2 * i + 2] = [[math.cos(a), -math.sin(a)],
                                                   [math.sin(a), math.cos(a)]]
        np.testing.assert_allclose(q[r, :128], R @ q[0, :128], atol=1e-12)


def test_rope_preserves_each_pair_norm():
    rows = _grid_rows(**TINY)
    qh, kh = RNG.standard_normal(128), RNG.standard_normal(128)
    q, k = oracle.qknorm_rope3d(_qkv_same_every_row(qh, kh, rows, 2), eps=1e-6, **TINY)
    for out in (q, k):
        n = np.hypot(out[:, 0::2], out[:, 1::2])
        np.testing.assert_allclose(n, np.broadcast_to(n[0], n.shape), rtol=1e-12)


def test_rope_audio_rows_are_1d_temporal():
    # audio row i behaves as the video position (t=i, h=0, w=0): audio row 1
    # (row 49) equals video row 24 = (1,0,0); audio row 0 equals row 0.
    rows = _grid_rows(**TINY)
    qh, kh = RNG.standard_normal(128), RNG.standard_normal(128)
    q, k = oracle.qknorm_rope3d(_qkv_same_every_row(qh, kh, rows, 2), eps=1e-6, **TINY)
    np.testing.assert_array_equal(q[49], q[24])
    np.testing.assert_array_equal(k[48], k[0])
    # audio row 7 (row 55): h and w sections untouched, t section rotated
    np.testing.assert_array_equal(q[55, 32:128], q[0, 32:128])
    assert np.max(np.abs(q[55, :32] - q[0, :32])) > 1e-3


@pytest.mark.parametrize("half", [False, True])
def test_rope_composition_adds_angles(half):
    # R(phi1) R(phi2) = R(phi1 + phi2): with eps = 0 and no gamma a head that
    # is already normalised passes QKNorm unchanged (rms 1), so
    # rotating audio row i1's output again as audio row i2 equals rotating
    # the input once as audio row i1 + i2 (positions (i, 0, 0))
    hd, nh, na = 128, 2, 12
    x = f32(RNG.standard_normal((1, 3 * nh * hd)))

    def rope_audio(inp, i):
        rows = np.repeat(inp, na, axis=0)
        q, k = oracle.qknorm_rope3d_ex(rows, 1, 1, 1, na - 1, nh, hd, (16, 24, 24), 0.0, 1e4,
                                       half)
        return q[1 + i], k[1 + i]  # row 0 is the single video row at (0, 0, 0)

    for i1, i2 in ((1, 2), (3, 4), (5, 5)):
        q1, k1 = rope_audio(x, i1)
        # fed back as fp32 (the oracle's input type): ~1e-7 relative rounding
        again = f32(np.concatenate([q1, k1, np.zeros(nh * hd)])[None, :])
        q12, k12 = rope_audio(again, i2)
        q_once, k_once = rope_audio(x, i1 + i2)
        np.testing.assert_allclose(q12, q_once, rtol=0, atol=1e-6)
        np.testing.assert_allclose(k12, k_once, rtol=0, atol=1e-6)


def test_rope_video_column_grid_is_1d_temporal():
    # H = W = 1: video row t sits at (t, 0, 0), exactly where an audio-only
    # sequence puts audio row t, so the two agree element by element (both
    # reduce to 1D RoPE on the t section)
    rows, nh, hd = 7, 2, 128
    qkv = f32(np.tile(RNG.standard_normal((1, 3 * nh * hd)), (rows, 1)))  # one row repeated
    for half in (False, True):
        qv, kv = oracle.qknorm_rope3d_ex(qkv, rows, 1, 1, 0, nh, hd, (16, 24, 24), 1e-6, 1e4,
                                         half)
        qa, ka = oracle.qknorm_rope3d_ex(qkv, 0, 0, 0, rows, nh, hd, (16, 24, 24), 1e-6, 1e4,
                                         half)
        np.testing.assert_array_equal(qv, qa)
        np.testing.assert_array_equal(kv, ka)
        # the same input row: row 3 differs from row 0 only by its rotation,
        # which touches the t section and nothing else
        assert np.abs(qv[3] - qv[0]).max() > 1e-3
        t_cols = np.r_[0:32] if not half else np.r_[0:16, 64:80]
        other = np.setdiff1d(np.arange(hd), t_cols)
        np.testing.assert_array_equal(qv[3, other], qv[0, other])


def test_rope_scores_depend_only_on_position_difference():
    # q.k per head after RoPE depends only on (dt, dh, dw) (RoFormer's
    # relative-position property), so equal displacements give equal scores.
    grid = dict(T=3, H=3, W=4, n_audio=0, n_heads=1, head_dim=128,
                sections=(16, 24, 24), theta=10000.0)
    rows = 36
    qh, kh = RNG.standard_normal(128), RNG.standard_normal(128)
    q, k = oracle.qknorm_rope3d(_qkv_same_every_row(qh, kh, rows, 1), eps=1e-6, **grid)

    def idx(t, h, w):
        return t * 12 + h * 4 + w

    groups = {}
    for a in range(rows):
        ta, ha, wa = a // 12, (a // 4) % 3, a % 4
        for b in range(rows):
            tb, hb, wb = b // 12, (b // 4) % 3, b % 4
            groups.setdefault((tb - ta, hb - ha, wb - wa), []).append(q[a] @ k[b])
    for delta, s in groups.items():
        np.testing.assert_allclose(s, s[0], rtol=0, atol=1e-10, err_msg=str(delta))
    vals = np.array([s[0] for s in groups.values()])
    assert np.unique(np.round(vals, 6)).size > 0.9 * len(vals)
    assert idx(2, 2, 3) == rows - 1


def test_qknorm_row_ids_and_row_stride():
    rows = _grid_rows(**TINY)
    qkv = f32(RNG.standard_normal((rows, 3 * 256 + 16)))
    q, k = oracle.qknorm_rope3d(qkv, eps=1e-6, **TINY)
    ids = np.array([55, 0, 23, 48], dtype=np.int64)
    qs, ks = oracle.qknorm_rope3d(qkv[ids], eps=1e-6, row_ids=ids, **TINY)
    np.testing.assert_array_equal(qs, q[ids])
    np.testing.assert_array_equal(ks, k[ids])


def test_qknorm_rejects_bad_sections():
    qkv = f32(np.ones((56, 768)))
    with pytest.raises(ValueError):
        oracle.qknorm_rope3d(qkv, 2, 4, 6, 8, 2, 128, (16, 24, 23), 1e-6, 1e4)


# ----------------------------------------------------------------------------
# Tolerance helper
# ----------------------------------------------------------------------------

def test_ulp_values():
    np.testing.assert_array_equal(oracle.ulp([1.0, 1.5, 3.0, 0.75, -8.0], oracle.BF16),
                                  [2.0 ** -7, 2.0 ** -7, 2.0 ** -6, 2.0 ** -8, 2.0 ** -4])
    np.testing.assert_array_equal(oracle.ulp([1.0, 0.1], oracle.F32),
                                  [2.0 ** -23, 2.0 ** -27])
    assert oracle.tolerance(0.0, oracle.BF16) == pytest.approx(1e-3)


# ----------------------------------------------------------------------------
# Fused gated residual + RMS-AdaLN
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("conv", [f32, bf16_bits], ids=["f32", "bf16"])
def test_fused_residual_norm_hand_worked(conv):
    h = _hand()
    hh = conv(np.stack([h["fused_h0"], h["fused_h1"]]))
    br = conv(np.stack([h["fused_b0"], h["fused_b1"]]))
    gate = conv(np.stack([h["fused_gate_video"], h["fused_gate_audio"]])[None])
    scale = conv(np.stack([h["scale_video"], h["scale_audio"]])[None])
    shift = conv(np.stack([h["shift_video"], h["shift_audio"]])[None])
    h_out, y = oracle.gate_residual_rms_adaln(hh, br, gate, scale, shift, L=2, n_video=1,
                                              eps=0.0)
    np.testing.assert_array_equal(h_out[0], h["fused_hout0"])
    np.testing.assert_array_equal(h_out[1], h["fused_hout1"])
    np.testing.assert_allclose(y[0], h["y0"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(y[1], h["y1"], rtol=0, atol=1e-14)
    _, yg = oracle.gate_residual_rms_adaln(hh, br, gate, scale, shift, L=2, n_video=1, eps=0.0,
                                           gamma=conv(h["gamma"]))
    np.testing.assert_allclose(yg[0], h["y0_gamma"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(yg[1], h["y1_gamma"], rtol=0, atol=1e-14)


def test_fused_residual_norm_closed_forms():
    # gate = 0: h_out is h exactly; with scale = shift = 0 and eps = 0 the
    # output has unit RMS; with scale = -1 the output is the shift.
    B, L, nv, D = 2, 5, 3, 32
    hh = f32(RNG.standard_normal((B * L, D)))
    br = f32(RNG.standard_normal((B * L, D)))
    z = f32(np.zeros((B, 2, D)))
    h_out, y = oracle.gate_residual_rms_adaln(hh, br, z, z, z, L=L, n_video=nv, eps=0.0)
    np.testing.assert_array_equal(h_out, hh.astype(np.float64))
    np.testing.assert_allclose(np.sqrt(np.mean(y ** 2, axis=1)), 1.0, rtol=1e-13)
    g = f32(RNG.standard_normal((B, 2, D)))
    shift = f32(np.array([[[10 * b + m + 1] * D for m in range(2)] for b in range(B)]))
    _, y = oracle.gate_residual_rms_adaln(hh, br, g, f32(np.full((B, 2, D), -1.0)), shift,
                                          L=L, n_video=nv, eps=1e-6)
    for row in range(B * L):
        b, r = divmod(row, L)
        assert np.all(y[row] == 10 * b + (0 if r < nv else 1) + 1)
    # h_out is linear in the gate: h_out(2g) - h_out(g) == h_out(g) - h_out(0)
    h1, _ = oracle.gate_residual_rms_adaln(hh, br, g, z, z, L=L, n_video=nv, eps=1e-6)
    h2, _ = oracle.gate_residual_rms_adaln(hh, br, f32(2 * g), z, z, L=L, n_video=nv, eps=1e-6)
    np.testing.assert_allclose(h2 - h1, h1 - hh.astype(np.float64), rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------
# First-Block-Cache change detector
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("conv", [f32, bf16_bits], ids=["f32", "bf16"])
def test_residual_change_hand_worked(conv):
    # sample 0: cur = [1, 2, -3, 4], prev = [1, 1, -1, 2]: |c-p| = 0,1,2,2 -> 5;
    #           |p| = 1+1+1+2 = 5 -> rel 1.0
    # sample 1: cur = prev = [0.5, -0.5, 0.25, 0] -> num 0, den 1.25, rel 0
    # batch: num 5, den 6.25, rel 0.8
    cur = conv([[1, 2, -3, 4], [0.5, -0.5, 0.25, 0]])
    prev = conv([[1, 1, -1, 2], [0.5, -0.5, 0.25, 0]])
    out = oracle.residual_change(cur, prev, B=2, L=1)
    np.testing.assert_array_equal(out, [[5, 5, 1.0], [0, 1.25, 0.0], [5, 6.25, 0.8]])


def test_residual_change_closed_forms():
    B, L, D = 3, 7, 16
    prev = f32(RNG.standard_normal((B * L, D)))
    # identical steps: zero change
    out = oracle.residual_change(prev, prev, B, L)
    np.testing.assert_array_equal(out[:, 0], 0.0)
    np.testing.assert_array_equal(out[:, 2], 0.0)
    # cur = (1 + a) * prev changes every element by |a * p|: rel = |a|; with
    # 1 + a a power of two the scaled values stay exact
    out = oracle.residual_change(f32(prev * 2.0), prev, B, L)
    np.testing.assert_allclose(out[:, 2], 1.0, rtol=1e-15)
    out = oracle.residual_change(f32(prev * 0.5), prev, B, L)
    np.testing.assert_allclose(out[:, 2], 0.5, rtol=1e-15)
    # cur = -prev: rel = 2
    out = oracle.residual_change(f32(-prev), prev, B, L)
    np.testing.assert_allclose(out[:, 2], 2.0, rtol=1e-15)
    # batch row sums the per-sample rows
    cur = f32(RNG.standard_normal((B * L, D)))
    out = oracle.residual_change(cur, prev, B, L)
    np.testing.assert_allclose(out[B, :2], out[:B, :2].sum(axis=0), rtol=1e-14)


def test_residual_change_zero_denominator():
    z = f32(np.zeros((2, 4)))
    o = f32(np.ones((2, 4)))
    out = oracle.residual_change(z, z, 2, 1)
    assert np.all(out[:, 2] == 0.0)
    out = oracle.residual_change(o, z, 2, 1)
    assert np.all(np.isinf(out[:, 2]))


# ----------------------------------------------------------------------------
# QKNorm + RoPE epilogue variants: half-split pairs, INT8 heads
# ----------------------------------------------------------------------------

def test_half_split_angles_match_hand_table():
    # first half of every head = 1, second half = 0: with eps = 0 the head
    # normalises to sqrt2 in the first half; pair i = (x[i], x[i+64]) becomes
    # sqrt2 (cos phi_i, sin phi_i) at elements (i, i + 64).
    pos, pairs = _positions()
    rows = _grid_rows(**TINY)
    hd = TINY["head_dim"]
    qh = np.concatenate([np.ones(hd // 2), np.zeros(hd // 2)])
    qkv = _qkv_same_every_row(qh, qh, rows, TINY["n_heads"])
    q, k = oracle.qknorm_rope3d_ex(qkv, eps=0.0, half_split=True, **TINY)
    s2 = math.sqrt(2.0)
    for r, p in pos.items():
        for i, (axis, freq) in pairs.items():
            phi = p[axis] * freq
            for out in (q, k):
                for head in range(TINY["n_heads"]):
                    a, b = out[r, head * hd + i], out[r, head * hd + i + hd // 2]
                    assert abs(math.hypot(a, b) - s2) < 1e-13
                    assert abs(_wrap(math.atan2(b, a) - phi)) < 1e-12, (r, i)


def test_half_split_is_complex_multiplication_and_flag_off_is_interleaved():
    rows = _grid_rows(**TINY)
    qh, kh = RNG.standard_normal(128), RNG.standard_normal(128)
    qkv = _qkv_same_every_row(qh, kh, rows, 2)
    q, _ = oracle.qknorm_rope3d_ex(qkv, eps=1e-6, half_split=True, **TINY)
    z0 = q[0, :64] + 1j * q[0, 64:128]
    for r in range(rows):
        rot = z0 * np.exp(1j * _closed_form_angles(r))
        np.testing.assert_allclose(q[r, :64], rot.real, atol=1e-12)
        np.testing.assert_allclose(q[r, 64:128], rot.imag, atol=1e-12)
    qi, ki = oracle.qknorm_rope3d_ex(qkv, eps=1e-6, half_split=False, **TINY)
    q0, k0 = oracle.qknorm_rope3d(qkv, eps=1e-6, **TINY)
    np.testing.assert_array_equal(qi, q0)
    np.testing.assert_array_equal(ki, k0)


def test_quantize_heads_hand_worked():
    # head 0: max |x| = 127 -> scale 1; -63.5 rounds half to even (-64),
    # 0.5 -> 0, 1.5 -> 2.  head 1: all zero -> scale 0, codes 0.
    x = np.array([[127.0, -63.5, 0.5, 1.5, 0.0, 0.0, 0.0, 0.0]])
    code, scale = oracle.quantize_heads(x, n_heads=2, head_dim=4)
    np.testing.assert_array_equal(code, [[127, -64, 0, 2, 0, 0, 0, 0]])
    np.testing.assert_array_equal(scale, [[1.0, 0.0]])
    # a head scaled by 2: same codes, scale 2/127 * 127 / 2... -> scale doubles
    code2, scale2 = oracle.quantize_heads(2 * x, n_heads=2, head_dim=4)
    np.testing.assert_array_equal(code2, code)
    np.testing.assert_array_equal(scale2, 2 * scale)


def test_quantize_heads_bounds_and_error():
    x = RNG.standard_normal((9, 3 * 16)) * np.linspace(0.1, 40, 9)[:, None]
    code, scale = oracle.quantize_heads(x, n_heads=3, head_dim=16)
    assert code.min() >= -127 and code.max() <= 127
    deq = code.reshape(9, 3, 16) * scale[:, :, None]
    err = np.abs(deq - x.reshape(9, 3, 16))
    assert np.all(err <= scale[:, :, None] / 2 + 1e-12)
    assert np.all(np.abs(code.reshape(9, 3, 16)).max(axis=2) == 127)


def test_half_split_identity_at_origin_gives_gamma():
    hd = 128
    gq = f32(1.0 + 0.1 * RNG.standard_normal(hd))
    gk = f32(1.0 + 0.1 * RNG.standard_normal(hd))
    qkv = _qkv_same_every_row(np.full(hd, 2.0), np.full(hd, -0.5), 1, 2)
    q, k = oracle.qknorm_rope3d_ex(qkv, 1, 1, 1, 0, 2, hd, (16, 24, 24), 0.0, 1e4, True,
                                   gamma_q=gq, gamma_k=gk)
    np.testing.assert_allclose(q[0], np.tile(gq.astype(np.float64), 2), rtol=1e-15)
    np.testing.assert_allclose(k[0], np.tile(-gk.astype(np.float64), 2), rtol=1e-15)


# ----------------------------------------------------------------------------
# GEMM + GELU
# ----------------------------------------------------------------------------

def test_gelu_tanh_closed_forms():
    x = np.array([0.0, 0.5, 1.0, 2.0, 3.0, 10.0])
    g = oracle.gelu_tanh(x)
    assert g[0] == 0.0
    # odd part: gelu(x) - gelu(-x) = x exactly for the tanh form
    np.testing.assert_allclose(g - oracle.gelu_tanh(-x), x, rtol=1e-15, atol=1e-15)
    # saturation: gelu(10) ~ 10, gelu(-10) ~ 0
    assert abs(g[-1] - 10.0) < 1e-7 and abs(oracle.gelu_tanh(-10.0)) < 1e-7
    # x = 1: sqrt(2/pi) * 1.044715 = 0.833554...; 0.5 * (1 + tanh(that)) = 0.841192
    assert abs(g[2] - 0.841192) < 1e-6


def test_gemm_gelu_brute_force_and_layout():
    rng = np.random.default_rng(5)
    M, N, K = 3, 4, 5
    A = f32(rng.standard_normal((M, K)))
    B = f32(rng.standard_normal((N, K)))
    bias = f32(rng.standard_normal(N))
    C = oracle.gemm_gelu(A, B, bias)
    for m in range(M):
        for n in range(N):
            s = sum(float(A[m, k]) * float(B[n, k]) for k in range(K)) + float(bias[n])
            g = 0.5 * s * (1 + math.tanh(math.sqrt(2 / math.pi) * (s + 0.044715 * s ** 3)))
            assert abs(C[m, n] - g) < 1e-12
    # B a permutation: C = gelu(A[:, perm] + bias) -- a transposed operand fails
    K = N = 6
    A = f32(rng.standard_normal((4, K)))
    perm = np.array([3, 0, 5, 1, 4, 2])
    P = np.zeros((N, K), dtype=np.float32)
    P[np.arange(N), perm] = 1.0
    np.testing.assert_allclose(oracle.gemm_gelu(A, P), oracle.gelu_tanh(A[:, perm]),
                               rtol=1e-15, atol=1e-15)
    # bias runs along N (one value per output column)
    z = f32(np.zeros((2, K)))
    b = f32(np.arange(N) - 2.5)
    np.testing.assert_allclose(oracle.gemm_gelu(z, P, b), np.tile(oracle.gelu_tanh(b), (2, 1)))


def test_widen_bf16_bits():
    np.testing.assert_array_equal(oracle.widen(np.array([0x3F80, 0xC000, 0x4049], np.uint16)),
                                  [1.0, -2.0, 3.140625])
