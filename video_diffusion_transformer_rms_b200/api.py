"""Tensor-level calls on top of the C ABI: take torch CUDA tensors, pass
their pointers, shapes and the current stream to libsol.  Marshalling only
(PyTorch allocates outputs when the caller does not pass them); the
arithmetic runs in libsol's kernels.
"""
from typing import Optional, Sequence, Tuple

import torch

from . import _abi

_DT = {torch.float32: _abi.SOL_F32, torch.bfloat16: _abi.SOL_BF16}


def _dtype(*ts) -> int:
    dts = {t.dtype for t in ts if t is not None}
    if len(dts) != 1:
        raise TypeError(f"all tensors must share one dtype, got {dts}")
    dt = dts.pop()
    if dt not in _DT:
        raise TypeError(f"dtype {dt} is not supported (float32 or bfloat16)")
    return _DT[dt]


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libsol takes CUDA tensors")
    return t.data_ptr()


def _expect(t: Optional[torch.Tensor], shape, name: str, like: torch.Tensor):
    """The library sees only pointers, so every tensor handed to it must be
    contiguous, of exactly this shape, and on the device of `like`."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous tensor of shape {tuple(shape)}, got "
                         f"{tuple(t.shape)}{'' if t.is_contiguous() else ' (not contiguous)'}")
    if t.device != like.device:
        raise ValueError(f"{name} is on {t.device}, the inputs on {like.device}")


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def rms_adaln(x: torch.Tensor, scale: torch.Tensor, shift: torch.Tensor, n_video: int,
              gamma: Optional[torch.Tensor] = None, eps: float = 1e-6,
              out: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """y = RMSNorm(x) * gamma * (1 + scale[b, m]) + shift[b, m]; x: [B, L, D],
    scale/shift: [B, 2, D]."""
    if x.dim() != 3 or not x.is_contiguous():
        raise ValueError("x must be a contiguous [B, L, D] tensor")
    B, L, D = x.shape
    for t, shape, name in ((scale, (B, 2, D), "scale"), (shift, (B, 2, D), "shift"),
                           (gamma, (D,), "gamma"), (out, (B, L, D), "out")):
        _expect(t, shape, name, x)
    y = torch.empty_like(x) if out is None else out
    _abi.check(_abi.sol_rms_adaln(_ptr(x), _ptr(y), _ptr(scale), _ptr(shift), _ptr(gamma),
                                  B, L, n_video, D, eps, _dtype(x, y, scale, shift, gamma),
                                  _stream(stream)))
    return y


def gate_residual(h: torch.Tensor, branch: torch.Tensor, gate: torch.Tensor, n_video: int,
                  out: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """out = h + gate[b, m] * branch; h/branch: [B, L, D], gate: [B, 2, D]."""
    if h.dim() != 3 or not h.is_contiguous():
        raise ValueError("h must be a contiguous [B, L, D] tensor")
    B, L, D = h.shape
    for t, shape, name in ((branch, (B, L, D), "branch"), (gate, (B, 2, D), "gate"),
                           (out, (B, L, D), "out")):
        _expect(t, shape, name, h)
    o = torch.empty_like(h) if out is None else out
    _abi.check(_abi.sol_gate_residual(_ptr(h), _ptr(branch), _ptr(gate), _ptr(o), B, L,
                                      n_video, D, _dtype(h, branch, gate, o), _stream(stream)))
    return o


def gate_residual_rms_adaln(h: torch.Tensor, branch: torch.Tensor, gate: torch.Tensor,
                            scale: torch.Tensor, shift: torch.Tensor, n_video: int,
                            gamma: Optional[torch.Tensor] = None, eps: float = 1e-6,
                            h_out: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                            stream: Optional[torch.cuda.Stream] = None
                            ) -> Tuple[torch.Tensor, torch.Tensor]:
    """h_out = h + gate[b, m] * branch; y = RMS-AdaLN(h_out) with scale/shift;
    returns (h_out, y).  Pass h_out=h to update the residual stream in place."""
    if h.dim() != 3 or not h.is_contiguous():
        raise ValueError("h must be a contiguous [B, L, D] tensor")
    B, L, D = h.shape
    for t, shape, name in ((branch, (B, L, D), "branch"), (gate, (B, 2, D), "gate"),
                           (scale, (B, 2, D), "scale"), (shift, (B, 2, D), "shift"),
                           (gamma, (D,), "gamma"), (h_out, (B, L, D), "h_out"),
                           (y, (B, L, D), "y")):
        _expect(t, shape, name, h)
    ho = torch.empty_like(h) if h_out is None else h_out
    yo = torch.empty_like(h) if y is None else y
    _abi.check(_abi.sol_gate_residual_rms_adaln(
        _ptr(h), _ptr(branch), _ptr(gate), _ptr(ho), _ptr(yo), _ptr(scale), _ptr(shift),
        _ptr(gamma), B, L, n_video, D, eps, _dtype(h, branch, gate, ho, yo, scale, shift, gamma),
        _stream(stream)))
    return ho, yo


def residual_change(cur: torch.Tensor, prev: torch.Tensor,
                    prev_out: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """First-Block-Cache change of a [B, L, D] residual against the previous
    step's: returns a [B + 1, 3] float64 CUDA tensor of (sum |cur - prev|,
    sum |prev|, their ratio) per sample and, in the last row, for the batch.
    With prev_out (may be prev itself) the cache is refreshed to cur in the
    same pass.  The workspace is allocated by PyTorch unless given."""
    if cur.dim() != 3 or not cur.is_contiguous():
        raise ValueError("cur must be a contiguous [B, L, D] tensor")
    B, L, D = cur.shape
    for t, shape, name in ((prev, (B, L, D), "prev"), (prev_out, (B, L, D), "prev_out"),
                           (out, (B + 1, 3), "out")):
        _expect(t, shape, name, cur)
    if out is not None and out.dtype != torch.float64:
        raise TypeError("out must be float64")
    if workspace is not None:
        _expect(workspace, (workspace.numel(),), "workspace", cur)
    need = _abi.sol_residual_change_workspace_bytes(B)
    ws = workspace if workspace is not None else torch.empty(
        max(need, 16), dtype=torch.uint8, device=cur.device)
    o = out if out is not None else torch.empty((B + 1, 3), dtype=torch.float64,
                                                device=cur.device)
    _abi.check(_abi.sol_residual_change(
        _ptr(cur), _ptr(prev), _ptr(prev_out), B, L, D, _ptr(o), _ptr(ws),
        ws.numel() * ws.element_size(), _dtype(cur, prev, prev_out), _stream(stream)))
    return o


class RopeTable:
    """A rotary table on the device (sol_rope_table): row p holds cos(p*f_i)
    for every rotary pair i, then sin(p*f_i), fp32, for positions
    0 .. n_pos-1.  Build it once per video shape; pass it as `table=` to
    qknorm_rope3d / qknorm_rope3d_ex."""

    def __init__(self, n_pos: int, head_dim: int, sections: Sequence[int] = (16, 24, 24),
                 theta: float = 10000.0, per_axis_freq: bool = False, device=None,
                 stream: Optional[torch.cuda.Stream] = None):
        nbytes = _abi.sol_rope_table_bytes(n_pos, head_dim)
        if nbytes == 0 and n_pos != 0:
            raise ValueError("n_pos must be >= 0 and head_dim even in [2, 256]")
        self.data = torch.empty(max(nbytes // 4, 4), dtype=torch.float32, device=device)
        self.n_pos, self.head_dim = n_pos, head_dim
        self.sections = tuple(int(x) for x in sections)
        self.theta, self.per_axis_freq = float(theta), bool(per_axis_freq)
        st, sh, sw = self.sections
        self.desc = _abi.RopeTable(self.data.data_ptr(), n_pos, head_dim, st, sh, sw, theta,
                                   int(self.per_axis_freq))
        _abi.check(_abi.sol_rope_table_build(self.desc, _stream(stream)))

    @classmethod
    def for_grid(cls, T: int, H: int, W: int, n_audio: int, head_dim: int, **kw):
        """A table covering every position of a T x H x W video grid plus
        n_audio audio tokens."""
        n = max(n_audio, max(T, H, W) if T * H * W > 0 else 0)
        return cls(n, head_dim, **kw)

    def check(self, head_dim: int, sections: Sequence[int], theta: float,
              per_axis_freq: bool = False):
        if (head_dim != self.head_dim or tuple(sections) != self.sections
                or float(theta) != self.theta or bool(per_axis_freq) != self.per_axis_freq):
            raise ValueError("the rotary table was built for other head_dim, sections, theta "
                             "or frequency rule")


def qknorm_rope3d(qkv: torch.Tensor, T: int, H: int, W: int, n_audio: int, n_heads: int,
                  head_dim: int, sections: Sequence[int] = (16, 24, 24),
                  gamma_q: Optional[torch.Tensor] = None,
                  gamma_k: Optional[torch.Tensor] = None, eps: float = 1e-6,
                  theta: float = 10000.0, q_out: Optional[torch.Tensor] = None,
                  k_out: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None,
                  table: Optional[RopeTable] = None
                  ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-head QKNorm + 3D RoPE of q and k in a merged qkv [B, L, >=2D]
    (row stride qkv.stride(1)); returns (q, k) as [B, L, D] views.  With
    `table` the (cos, sin) come from that rotary table (sol_qknorm_rope3d_tab)
    instead of being computed per row."""
    if qkv.dim() != 3 or qkv.stride(2) != 1 or qkv.stride(0) != qkv.shape[1] * qkv.stride(1):
        raise ValueError("qkv must be [B, L, C] with unit column stride and packed rows")
    B, L, _ = qkv.shape
    D = n_heads * head_dim
    if L != T * H * W + n_audio:
        raise ValueError("L must equal T*H*W + n_audio")
    for t, name in ((gamma_q, "gamma_q"), (gamma_k, "gamma_k")):
        _expect(t, (head_dim,), name, qkv)
    if q_out is None and k_out is None:
        buf = torch.empty((B, L, 2 * D), dtype=qkv.dtype, device=qkv.device)
        q_out, k_out = buf[..., :D], buf[..., D:]
    elif q_out is None or k_out is None:
        raise ValueError("pass both q_out and k_out, or neither")
    if q_out.stride() != k_out.stride() or q_out.stride(2) != 1:
        raise ValueError("q_out and k_out must share a row stride with unit column stride")
    for t, name in ((q_out, "q_out"), (k_out, "k_out")):
        if tuple(t.shape) != (B, L, D) or t.stride(0) != L * t.stride(1):
            raise ValueError(f"{name} must be a [B, L, D] view with packed rows")
        if t.device != qkv.device:
            raise ValueError(f"{name} is on {t.device}, qkv on {qkv.device}")
    ld_out = q_out.stride(1)
    st, sh, sw = sections
    dt = _dtype(qkv, q_out, k_out, gamma_q, gamma_k)
    if table is not None:
        table.check(head_dim, sections, theta)
        if table.data.device != qkv.device:
            raise ValueError(f"the rotary table is on {table.data.device}, qkv on {qkv.device}")
        _abi.check(_abi.sol_qknorm_rope3d_tab(
            _ptr(qkv), qkv.stride(1), _ptr(q_out), _ptr(k_out), ld_out, _ptr(gamma_q),
            _ptr(gamma_k), table.desc, B, T, H, W, n_audio, n_heads, eps, dt, _stream(stream)))
    else:
        _abi.check(_abi.sol_qknorm_rope3d(
            _ptr(qkv), qkv.stride(1), _ptr(q_out), _ptr(k_out), ld_out, _ptr(gamma_q),
            _ptr(gamma_k), B, T, H, W, n_audio, n_heads, head_dim, st, sh, sw, eps, theta, dt,
            _stream(stream)))
    return q_out, k_out


def qknorm_rope3d_ex(qkv: torch.Tensor, T: int, H: int, W: int, n_audio: int, n_heads: int,
                     head_dim: int, sections: Sequence[int] = (16, 24, 24),
                     gamma_q: Optional[torch.Tensor] = None,
                     gamma_k: Optional[torch.Tensor] = None, eps: float = 1e-6,
                     theta: float = 10000.0, layout: str = "bshd", half_split: bool = False,
                     int8: bool = False, per_axis_freq: bool = False, quantize_v: bool = False,
                     stream: Optional[torch.cuda.Stream] = None,
                     table: Optional[RopeTable] = None):
    """QKNorm + 3D RoPE epilogue variants (bf16 input).  layout "bshd" gives
    q, k as [B, L, H, hd]; "bhsd" as attention's [B, H, L, hd].  half_split
    pairs element i with i + hd/2; per_axis_freq gives each rotary section a
    frequency ladder of its own.  int8 returns (q, k, q_scale, k_scale): int8
    codes in the chosen layout and scales fp32 [B, L, H]; with quantize_v
    also (v, v_scale), v quantised as it stands; else (q, k) in bf16.  With
    `table` the (cos, sin) come from that rotary table
    (sol_qknorm_rope3d_ex_tab)."""
    if qkv.dim() != 3 or qkv.stride(2) != 1 or qkv.stride(0) != qkv.shape[1] * qkv.stride(1):
        raise ValueError("qkv must be [B, L, C] with unit column stride and packed rows")
    if quantize_v and not int8:
        raise ValueError("quantize_v needs int8=True")
    B, L, _ = qkv.shape
    if L != T * H * W + n_audio:
        raise ValueError("L must equal T*H*W + n_audio")
    for t, name in ((gamma_q, "gamma_q"), (gamma_k, "gamma_k")):
        _expect(t, (head_dim,), name, qkv)
    odt = torch.int8 if int8 else qkv.dtype
    if layout == "bshd":
        shape = (B, L, n_heads, head_dim)
        strides = (L * n_heads * head_dim, n_heads * head_dim, head_dim)
    elif layout == "bhsd":
        shape = (B, n_heads, L, head_dim)
        strides = (n_heads * L * head_dim, head_dim, L * head_dim)
    else:
        raise ValueError("layout must be 'bshd' or 'bhsd'")
    q = torch.empty(shape, dtype=odt, device=qkv.device)
    k = torch.empty(shape, dtype=odt, device=qkv.device)
    qs = ks = v = vs = None
    if int8:
        qs = torch.empty((B, L, n_heads), dtype=torch.float32, device=qkv.device)
        ks = torch.empty((B, L, n_heads), dtype=torch.float32, device=qkv.device)
    if quantize_v:
        v = torch.empty(shape, dtype=odt, device=qkv.device)
        vs = torch.empty((B, L, n_heads), dtype=torch.float32, device=qkv.device)
    lay = _abi.QkLayout(strides[0], strides[1], strides[2], int(bool(half_split)),
                        int(bool(int8)), _ptr(qs), _ptr(ks), int(bool(per_axis_freq)), 0,
                        _ptr(v), _ptr(vs))
    st, sh, sw = sections
    dt = _dtype(qkv, gamma_q, gamma_k)
    if table is not None:
        table.check(head_dim, sections, theta, per_axis_freq)
        if table.data.device != qkv.device:
            raise ValueError(f"the rotary table is on {table.data.device}, qkv on {qkv.device}")
        _abi.check(_abi.sol_qknorm_rope3d_ex_tab(
            _ptr(qkv), qkv.stride(1), _ptr(q), _ptr(k), lay, _ptr(gamma_q), _ptr(gamma_k),
            table.desc, B, T, H, W, n_audio, n_heads, eps, dt, _stream(stream)))
    else:
        _abi.check(_abi.sol_qknorm_rope3d_ex(
            _ptr(qkv), qkv.stride(1), _ptr(q), _ptr(k), lay, _ptr(gamma_q), _ptr(gamma_k), B, T,
            H, W, n_audio, n_heads, head_dim, st, sh, sw, eps, theta, dt, _stream(stream)))
    if quantize_v:
        return q, k, qs, ks, v, vs
    return (q, k, qs, ks) if int8 else (q, k)


def gemm_gelu(A: torch.Tensor, B: torch.Tensor, bias: Optional[torch.Tensor] = None,
              out: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """C = gelu_tanh(A @ B.T + bias) on the tensor cores; A [M, K], B [N, K]
    (a Linear weight), bias [N], all bf16; returns C [M, N] bf16."""
    if A.dim() != 2 or B.dim() != 2 or A.shape[1] != B.shape[1]:
        raise ValueError("A must be [M, K] and B [N, K]")
    if not (A.is_contiguous() and B.is_contiguous()):
        raise ValueError("A and B must be contiguous")
    M, K = A.shape
    N = B.shape[0]
    _expect(B, (N, K), "B", A)
    _expect(bias, (N,), "bias", A)
    _expect(out, (M, N), "out", A)
    C = torch.empty((M, N), dtype=A.dtype, device=A.device) if out is None else out
    need = _abi.sol_gemm_gelu_workspace_bytes(M, N, K)
    ws = torch.empty(need, dtype=torch.uint8, device=A.device) if need else None
    _dtype(A, B, bias, C)
    if A.dtype != torch.bfloat16:
        raise TypeError("sol_gemm_gelu takes bf16 tensors")
    _abi.check(_abi.sol_gemm_gelu(_ptr(A), _ptr(B), _ptr(bias), _ptr(C), M, N, K, _ptr(ws),
                                  need, _stream(stream)))
    return C
