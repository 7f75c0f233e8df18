"""fp64 CPU oracle for fused RMS-AdaLN, the AdaLN-gated residual and per-head
QKNorm + 3D multimodal RoPE.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg, never by the product package.  It shares no
code with the CUDA library.  The arithmetic lives in sol_oracle.c; this
module only loads it and passes numpy arrays.

Inputs are numpy arrays in the I/O dtype: float32, or uint16 holding bf16
bit patterns.  Outputs are float64 arrays (unrounded oracle values).
"""
import ctypes
import os

import numpy as np

from . import build as _build

F32 = 0
BF16 = 1

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        d = ctypes.c_double
        i = ctypes.c_int
        lib.oracle_rms_adaln.argtypes = [p, p, p, p, p, i64, i64, i64, i64, d, i, p]
        lib.oracle_rms_adaln.restype = i
        lib.oracle_gate_residual.argtypes = [p, p, p, p, i64, i64, i64, i64, i, p]
        lib.oracle_gate_residual.restype = i
        lib.oracle_gate_residual_rms_adaln.argtypes = [p, p, p, p, p, p, p, i64, i64, i64, i64,
                                                       d, i, p, p]
        lib.oracle_gate_residual_rms_adaln.restype = i
        lib.oracle_residual_change.argtypes = [p, p, i64, i64, i64, i, p]
        lib.oracle_residual_change.restype = i
        lib.oracle_qknorm_rope3d_ex.argtypes = [p, i64, p, p, p, i64, i64, i64, i64,
                                                i64, i64, i64, i64, i64, i64, d, d,
                                                i, i, i, p, p]
        lib.oracle_qknorm_rope3d_ex.restype = i
        lib.oracle_quantize_heads.argtypes = [p, i64, i64, i64, p, p]
        lib.oracle_quantize_heads.restype = i
        lib.oracle_qknorm_rope3d.argtypes = [p, i64, p, p, p, i64, i64, i64, i64,
                                             i64, i64, i64, i64, i64, i64, d, d,
                                             i, p, p]
        lib.oracle_qknorm_rope3d.restype = i
        _lib = lib
    return _lib


def _dtype_code(*arrays):
    codes = set()
    for a in arrays:
        if a is None:
            continue
        if a.dtype == np.float32:
            codes.add(F32)
        elif a.dtype == np.uint16:
            codes.add(BF16)
        else:
            raise TypeError(f"oracle inputs are float32 or uint16 (bf16 bits), got {a.dtype}")
    if len(codes) != 1:
        raise TypeError("oracle inputs must share one dtype")
    return codes.pop()


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a):
    return None if a is None else np.ascontiguousarray(a)


def _rows(row_ids, n_default):
    if row_ids is None:
        return None, n_default
    r = np.ascontiguousarray(row_ids, dtype=np.int64)
    return r, int(r.shape[0])


def rms_adaln(x, scale, shift, L, n_video, eps, gamma=None, row_ids=None):
    """x: [n_rows, D]; scale, shift: [B, 2, D]; gamma: [D] or None."""
    x, scale, shift, gamma = _c(x), _c(scale), _c(shift), _c(gamma)
    D = x.shape[-1]
    x2 = x.reshape(-1, D)
    rid, n = _rows(row_ids, x2.shape[0])
    if n != x2.shape[0]:
        raise ValueError("row_ids length must match the rows of x")
    y = np.empty((n, D), dtype=np.float64)
    rc = _load().oracle_rms_adaln(_ptr(x2), _ptr(scale), _ptr(shift), _ptr(gamma),
                                  _ptr(rid), n, L, n_video, D, eps,
                                  _dtype_code(x, scale, shift, gamma), _ptr(y))
    if rc != 0:
        raise ValueError("oracle_rms_adaln rejected its arguments")
    return y.reshape(x.shape)


def gate_residual(h, branch, gate, L, n_video, row_ids=None):
    """h, branch: [n_rows, D]; gate: [B, 2, D]."""
    h, branch, gate = _c(h), _c(branch), _c(gate)
    D = h.shape[-1]
    h2, b2 = h.reshape(-1, D), branch.reshape(-1, D)
    rid, n = _rows(row_ids, h2.shape[0])
    if n != h2.shape[0] or b2.shape != h2.shape:
        raise ValueError("h, branch and row_ids must agree")
    out = np.empty((n, D), dtype=np.float64)
    rc = _load().oracle_gate_residual(_ptr(h2), _ptr(b2), _ptr(gate), _ptr(rid), n, L,
                                      n_video, D, _dtype_code(h, branch, gate), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_gate_residual rejected its arguments")
    return out.reshape(h.shape)


def gate_residual_rms_adaln(h, branch, gate, scale, shift, L, n_video, eps, gamma=None,
                            row_ids=None):
    """h, branch: [n_rows, D]; gate, scale, shift: [B, 2, D]; returns (h_out, y)."""
    h, branch, gate, scale, shift, gamma = (_c(a) for a in (h, branch, gate, scale, shift, gamma))
    D = h.shape[-1]
    h2, b2 = h.reshape(-1, D), branch.reshape(-1, D)
    rid, n = _rows(row_ids, h2.shape[0])
    if n != h2.shape[0] or b2.shape != h2.shape:
        raise ValueError("h, branch and row_ids must agree")
    h_out = np.empty((n, D), dtype=np.float64)
    y = np.empty((n, D), dtype=np.float64)
    rc = _load().oracle_gate_residual_rms_adaln(
        _ptr(h2), _ptr(b2), _ptr(gate), _ptr(scale), _ptr(shift), _ptr(gamma), _ptr(rid), n, L,
        n_video, D, eps, _dtype_code(h, branch, gate, scale, shift, gamma), _ptr(h_out), _ptr(y))
    if rc != 0:
        raise ValueError("oracle_gate_residual_rms_adaln rejected its arguments")
    return h_out.reshape(h.shape), y.reshape(h.shape)


def residual_change(cur, prev, B, L):
    """cur, prev: [B*L, D] (or [B, L, D]); returns [B + 1, 3] (num, den, rel),
    the last row for the whole batch."""
    cur, prev = _c(cur), _c(prev)
    if cur.shape != prev.shape:
        raise ValueError("cur and prev must have one shape")
    D = cur.shape[-1]
    if cur.size != B * L * D:
        raise ValueError("cur must hold B*L rows")
    out = np.empty((B + 1, 3), dtype=np.float64)
    rc = _load().oracle_residual_change(_ptr(cur), _ptr(prev), B, L, D, _dtype_code(cur, prev),
                                        _ptr(out))
    if rc != 0:
        raise ValueError("oracle_residual_change rejected its arguments")
    return out


def qknorm_rope3d(qkv, T, H, W, n_audio, n_heads, head_dim, sections, eps, theta,
                  gamma_q=None, gamma_k=None, row_ids=None):
    """qkv: [n_rows, >= 2*D] (q, k, then anything); returns (q, k) [n_rows, D]."""
    qkv, gamma_q, gamma_k = _c(qkv), _c(gamma_q), _c(gamma_k)
    D = n_heads * head_dim
    q2 = qkv.reshape(-1, qkv.shape[-1])
    ld = q2.shape[1]
    rid, n = _rows(row_ids, q2.shape[0])
    if n != q2.shape[0]:
        raise ValueError("row_ids length must match the rows of qkv")
    q = np.empty((n, D), dtype=np.float64)
    k = np.empty((n, D), dtype=np.float64)
    st, sh, sw = sections
    rc = _load().oracle_qknorm_rope3d(_ptr(q2), ld, _ptr(gamma_q), _ptr(gamma_k), _ptr(rid),
                                      n, T, H, W, n_audio, n_heads, head_dim, st, sh, sw,
                                      eps, theta, _dtype_code(qkv, gamma_q, gamma_k),
                                      _ptr(q), _ptr(k))
    if rc != 0:
        raise ValueError("oracle_qknorm_rope3d rejected its arguments")
    return q, k


def qknorm_rope3d_ex(qkv, T, H, W, n_audio, n_heads, head_dim, sections, eps, theta,
                     half_split, gamma_q=None, gamma_k=None, row_ids=None, per_axis=False):
    """qknorm_rope3d with a rotary pair layout flag (half_split: pair i is
    elements (i, i + head_dim/2)) and a frequency ladder flag (per_axis: pair
    j of a section of s pairs turns at theta^(-j/s), each axis with a ladder
    of its own)."""
    qkv, gamma_q, gamma_k = _c(qkv), _c(gamma_q), _c(gamma_k)
    D = n_heads * head_dim
    q2 = qkv.reshape(-1, qkv.shape[-1])
    rid, n = _rows(row_ids, q2.shape[0])
    if n != q2.shape[0]:
        raise ValueError("row_ids length must match the rows of qkv")
    q = np.empty((n, D), dtype=np.float64)
    k = np.empty((n, D), dtype=np.float64)
    st, sh, sw = sections
    rc = _load().oracle_qknorm_rope3d_ex(_ptr(q2), q2.shape[1], _ptr(gamma_q), _ptr(gamma_k),
                                         _ptr(rid), n, T, H, W, n_audio, n_heads, head_dim, st,
                                         sh, sw, eps, theta, int(bool(half_split)),
                                         int(bool(per_axis)), _dtype_code(qkv, gamma_q, gamma_k),
                                         _ptr(q), _ptr(k))
    if rc != 0:
        raise ValueError("oracle_qknorm_rope3d_ex rejected its arguments")
    return q, k


def quantize_heads(x, n_heads, head_dim):
    """Symmetric per-head INT8 codes of x [n_rows, n_heads*head_dim] (fp64):
    returns (codes int32 [n_rows, D], scales fp64 [n_rows, n_heads])."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    n = x.shape[0]
    code = np.empty(x.shape, dtype=np.int32)
    scale = np.empty((n, n_heads), dtype=np.float64)
    rc = _load().oracle_quantize_heads(_ptr(x), n, n_heads, head_dim, _ptr(code), _ptr(scale))
    if rc != 0:
        raise ValueError("oracle_quantize_heads rejected its arguments")
    return code, scale


def widen(a):
    """Exact float64 values of an oracle input array (float32, or uint16 bf16 bits)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if a.dtype == np.float32:
        return a.astype(np.float64)
    raise TypeError(f"unsupported oracle input dtype {a.dtype}")


def gelu_tanh(x):
    """GELU, tanh form (Hendrycks & Gimpel): 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def gemm_gelu(A, B, bias=None):
    """gelu_tanh(A @ B.T + bias) in fp64; A [M, K], B [N, K], bias [N]; the
    matmul is numpy's (a library primitive), everything else is spelled out."""
    x = widen(A) @ widen(B).T
    if bias is not None:
        x = x + widen(bias)[None, :]
    return gelu_tanh(x)


def ulp(v, dtype):
    """Unit in the last place of the I/O dtype at the (fp64) value v.

    bf16 has 8 significand bits (7 stored): ulp = 2^(e-7); fp32: 2^(e-23),
    e = floor(log2|v|) clamped below at -126 (the normal range).
    """
    v = np.abs(np.asarray(v, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(v > 0, v, 1.0)))
    e = np.where(v > 0, np.maximum(e, -126.0), -126.0)
    mant = 7 if dtype == BF16 else 23
    return np.exp2(e - mant)


def tolerance(v, dtype, n_ulp=2.0, abs_tol=1e-3):
    """Per-element bound |gpu - v| <= n_ulp * ulp(v) + abs_tol."""
    return n_ulp * ulp(v, dtype) + abs_tol
