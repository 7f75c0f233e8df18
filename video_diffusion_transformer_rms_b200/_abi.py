"""ctypes binding of libsol (include/sol.h): the same entry points, same
names, same argument order.  Argument marshalling only; every step of the
computation runs in the CUDA kernels of libsol.so.

The library must have been built (python -m
video_diffusion_transformer_rms_b200.build, or __graft_entry__.build()); if
it is missing, the first call raises ImportError.  There is no fallback.
"""
import ctypes
import os
import re
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libsol.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "sol.h")

SOL_OK = 0
SOL_ERR_INVALID_ARG = 1
SOL_ERR_MISALIGNED = 2
SOL_ERR_UNSUPPORTED = 3
SOL_ERR_CUDA = 4

SOL_F32 = 0
SOL_BF16 = 1

class QkLayout(ctypes.Structure):
    """sol_qk_layout of include/sol.h."""
    _fields_ = [("stride_b", ctypes.c_int64), ("stride_row", ctypes.c_int64),
                ("stride_head", ctypes.c_int64), ("half_split", ctypes.c_int32),
                ("int8_out", ctypes.c_int32), ("q_scale", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("per_axis_freq", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("v_out", ctypes.c_void_p),
                ("v_scale", ctypes.c_void_p)]


class RopeTable(ctypes.Structure):
    """sol_rope_table of include/sol.h: a rotary table's device buffer and the
    fields it was (or will be) built from."""
    _fields_ = [("data", ctypes.c_void_p), ("n_pos", ctypes.c_int64),
                ("head_dim", ctypes.c_int64), ("sec_t", ctypes.c_int64),
                ("sec_h", ctypes.c_int64), ("sec_w", ctypes.c_int64),
                ("theta", ctypes.c_float), ("per_axis_freq", ctypes.c_int32)]


_lock = threading.Lock()
_lib = None


class SolError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{status_string(status)}: {message}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libsol.so once and declare its prototypes."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"libsol.so is not built ({LIB_PATH}); run "
                "`python -m video_diffusion_transformer_rms_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        p, i64, f, i = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int
        L.sol_rms_adaln.argtypes = [p, p, p, p, p, i64, i64, i64, i64, f, i, p]
        L.sol_rms_adaln.restype = i
        L.sol_gate_residual.argtypes = [p, p, p, p, i64, i64, i64, i64, i, p]
        L.sol_gate_residual.restype = i
        L.sol_gate_residual_rms_adaln.argtypes = [p, p, p, p, p, p, p, p, i64, i64, i64, i64, f,
                                                  i, p]
        L.sol_gate_residual_rms_adaln.restype = i
        L.sol_residual_change.argtypes = [p, p, p, i64, i64, i64, p, p, ctypes.c_size_t, i, p]
        L.sol_residual_change.restype = i
        L.sol_residual_change_workspace_bytes.argtypes = [i64]
        L.sol_residual_change_workspace_bytes.restype = ctypes.c_size_t
        L.sol_residual_change_noalloc.argtypes = [p, p, p, i64, i64, i64, p, i, p]
        L.sol_residual_change_noalloc.restype = i
        L.sol_qknorm_rope3d_ex.argtypes = [p, i64, p, p, ctypes.POINTER(QkLayout), p, p, i64,
                                           i64, i64, i64, i64, i64, i64, i64, i64, i64, f, f,
                                           i, p]
        L.sol_qknorm_rope3d_ex.restype = i
        L.sol_gemm_gelu.argtypes = [p, p, p, p, i64, i64, i64, p, ctypes.c_size_t, p]
        L.sol_gemm_gelu.restype = i
        L.sol_gemm_gelu_workspace_bytes.argtypes = [i64, i64, i64]
        L.sol_gemm_gelu_workspace_bytes.restype = ctypes.c_size_t
        L.sol_qknorm_rope3d.argtypes = [p, i64, p, p, i64, p, p, i64, i64, i64, i64, i64,
                                        i64, i64, i64, i64, i64, f, f, i, p]
        L.sol_qknorm_rope3d.restype = i
        L.sol_rope_table_bytes.argtypes = [i64, i64]
        L.sol_rope_table_bytes.restype = ctypes.c_size_t
        L.sol_rope_table_build.argtypes = [ctypes.POINTER(RopeTable), p]
        L.sol_rope_table_build.restype = i
        L.sol_qknorm_rope3d_tab.argtypes = [p, i64, p, p, i64, p, p, ctypes.POINTER(RopeTable),
                                            i64, i64, i64, i64, i64, i64, f, i, p]
        L.sol_qknorm_rope3d_tab.restype = i
        L.sol_qknorm_rope3d_ex_tab.argtypes = [p, i64, p, p, ctypes.POINTER(QkLayout), p, p,
                                               ctypes.POINTER(RopeTable), i64, i64, i64, i64,
                                               i64, i64, f, i, p]
        L.sol_qknorm_rope3d_ex_tab.restype = i
        L.sol_status_string.argtypes = [i]
        L.sol_status_string.restype = ctypes.c_char_p
        L.sol_last_error.argtypes = []
        L.sol_last_error.restype = ctypes.c_char_p
        L.sol_version.argtypes = []
        L.sol_version.restype = i
        _lib = L
    return _lib


def header_symbols():
    """Names of the functions include/sol.h declares."""
    with open(HEADER) as fh:
        text = fh.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(sol_\w+)\s*\(", text, re.M)))


def status_string(status: int) -> str:
    return lib().sol_status_string(status).decode()


def last_error() -> str:
    return lib().sol_last_error().decode()


def check(status: int) -> None:
    if status != SOL_OK:
        raise SolError(status, last_error())


def sol_rms_adaln(x, y, scale, shift, gamma, B, L, n_video, D, eps, dtype, stream) -> int:
    return lib().sol_rms_adaln(x, y, scale, shift, gamma, B, L, n_video, D, eps, dtype, stream)


def sol_gate_residual(h, branch, gate, out, B, L, n_video, D, dtype, stream) -> int:
    return lib().sol_gate_residual(h, branch, gate, out, B, L, n_video, D, dtype, stream)


def sol_gate_residual_rms_adaln(h, branch, gate, h_out, y, scale, shift, gamma, B, L, n_video,
                                D, eps, dtype, stream) -> int:
    return lib().sol_gate_residual_rms_adaln(h, branch, gate, h_out, y, scale, shift, gamma, B,
                                             L, n_video, D, eps, dtype, stream)


def sol_residual_change(cur, prev, prev_out, B, L, D, out, workspace, workspace_bytes, dtype,
                        stream) -> int:
    return lib().sol_residual_change(cur, prev, prev_out, B, L, D, out, workspace,
                                     workspace_bytes, dtype, stream)


def sol_residual_change_workspace_bytes(B) -> int:
    return lib().sol_residual_change_workspace_bytes(B)


def sol_residual_change_noalloc(cur, prev, prev_out, B, L, D, out, dtype, stream) -> int:
    """sol_residual_change with its scratch inside libsol (B <= 16): for
    callers that cannot allocate device memory."""
    return lib().sol_residual_change_noalloc(cur, prev, prev_out, B, L, D, out, dtype, stream)


def sol_qknorm_rope3d(qkv, ld_qkv, q_out, k_out, ld_out, gamma_q, gamma_k, B, T, H, W,
                      n_audio, n_heads, head_dim, sec_t, sec_h, sec_w, eps, theta, dtype,
                      stream) -> int:
    return lib().sol_qknorm_rope3d(qkv, ld_qkv, q_out, k_out, ld_out, gamma_q, gamma_k, B, T,
                                   H, W, n_audio, n_heads, head_dim, sec_t, sec_h, sec_w,
                                   eps, theta, dtype, stream)


def sol_qknorm_rope3d_ex(qkv, ld_qkv, q_out, k_out, layout, gamma_q, gamma_k, B, T, H, W,
                         n_audio, n_heads, head_dim, sec_t, sec_h, sec_w, eps, theta, dtype,
                         stream) -> int:
    """layout: a QkLayout (or None, which the library rejects)."""
    ref = ctypes.byref(layout) if layout is not None else None
    return lib().sol_qknorm_rope3d_ex(qkv, ld_qkv, q_out, k_out, ref, gamma_q, gamma_k, B, T,
                                      H, W, n_audio, n_heads, head_dim, sec_t, sec_h, sec_w,
                                      eps, theta, dtype, stream)


def _ref(x):
    return ctypes.byref(x) if x is not None else None


def sol_rope_table_bytes(n_pos, head_dim) -> int:
    return lib().sol_rope_table_bytes(n_pos, head_dim)


def sol_rope_table_build(tab, stream) -> int:
    """tab: a RopeTable (or None, which the library rejects)."""
    return lib().sol_rope_table_build(_ref(tab), stream)


def sol_qknorm_rope3d_tab(qkv, ld_qkv, q_out, k_out, ld_out, gamma_q, gamma_k, tab, B, T, H, W,
                          n_audio, n_heads, eps, dtype, stream) -> int:
    return lib().sol_qknorm_rope3d_tab(qkv, ld_qkv, q_out, k_out, ld_out, gamma_q, gamma_k,
                                       _ref(tab), B, T, H, W, n_audio, n_heads, eps, dtype,
                                       stream)


def sol_qknorm_rope3d_ex_tab(qkv, ld_qkv, q_out, k_out, layout, gamma_q, gamma_k, tab, B, T, H,
                             W, n_audio, n_heads, eps, dtype, stream) -> int:
    return lib().sol_qknorm_rope3d_ex_tab(qkv, ld_qkv, q_out, k_out, _ref(layout), gamma_q,
                                          gamma_k, _ref(tab), B, T, H, W, n_audio, n_heads, eps,
                                          dtype, stream)


def sol_gemm_gelu(A, B, bias, C, M, N, K, workspace, workspace_bytes, stream) -> int:
    return lib().sol_gemm_gelu(A, B, bias, C, M, N, K, workspace, workspace_bytes, stream)


def sol_gemm_gelu_workspace_bytes(M, N, K) -> int:
    return lib().sol_gemm_gelu_workspace_bytes(M, N, K)


def sol_status_string(status: int) -> str:
    return status_string(status)


def sol_last_error() -> str:
    return last_error()


def sol_version() -> int:
    return lib().sol_version()
