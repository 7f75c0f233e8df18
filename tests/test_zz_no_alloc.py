"""The allocation-free change detector, sol_residual_change_noalloc.

It serves callers that cannot call cudaMalloc: hosts whose device memory
already belongs to their own pool or framework allocator, hot loops that
must not pay cudaMalloc's implicit synchronisation, plain-C plug-ins with no
allocator at hand.  It keeps its partial sums in an array inside libsol
instead of a caller workspace.  This test calls it through the C ABI twice in
a row, on two different inputs, and checks each result against the
workspace entry point sol_residual_change within the tolerance the parity
tests use (relative 1e-5).  The inputs and outputs here are allocated by the
test; the entry point itself allocates nothing.
"""
import ctypes

import numpy as np
import pytest
import torch

from video_diffusion_transformer_rms_b200 import _abi

pytestmark = pytest.mark.gpu


def _inputs(B, L, D, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    prev = torch.randn((B, L, D), generator=g, device="cuda").to(torch.bfloat16)
    noise = torch.randn((B, L, D), generator=g, device="cuda")
    cur = (prev.float() * (1.0 + 0.05 * noise)).to(torch.bfloat16)
    return cur, prev


def _with_workspace(cur, prev, prev_out=None):
    B, L, D = cur.shape
    ws = torch.empty(_abi.sol_residual_change_workspace_bytes(B), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((B + 1, 3), dtype=torch.float64, device="cuda")
    _abi.check(_abi.sol_residual_change(
        cur.data_ptr(), prev.data_ptr(), None if prev_out is None else prev_out.data_ptr(),
        B, L, D, out.data_ptr(), ws.data_ptr(), ws.numel(), _abi.SOL_BF16,
        torch.cuda.current_stream().cuda_stream))
    return out


def _no_alloc(cur, prev, prev_out=None):
    B, L, D = cur.shape
    out = torch.empty((B + 1, 3), dtype=torch.float64, device="cuda")
    _abi.check(_abi.sol_residual_change_noalloc(
        cur.data_ptr(), prev.data_ptr(), None if prev_out is None else prev_out.data_ptr(),
        B, L, D, out.data_ptr(), _abi.SOL_BF16, torch.cuda.current_stream().cuda_stream))
    return out


def _close(got, want):
    g, w = got.cpu().numpy(), want.cpu().numpy()
    np.testing.assert_allclose(g, w, rtol=1e-5, atol=1e-30)


def test_no_alloc_matches_workspace_entry_point_twice_in_a_row():
    assert torch.cuda.is_available(), "this test needs a CUDA device"
    _abi.lib()
    cases = [_inputs(2, 4099, 5120, seed=1), _inputs(3, 1500, 3072, seed=2)]
    wants = [_with_workspace(c, p) for c, p in cases]
    gots = [_no_alloc(c, p) for c, p in cases]  # two calls in a row
    torch.cuda.synchronize()
    for got, want in zip(gots, wants):
        _close(got, want)
        assert 0.0 < float(want[-1, 2]) < 1.0


def test_no_alloc_cache_refresh_and_limit():
    cur, prev = _inputs(1, 777, 2048, seed=3)
    want = _with_workspace(cur, prev)
    refreshed = torch.empty_like(prev)
    got = _no_alloc(cur, prev, prev_out=refreshed)
    torch.cuda.synchronize()
    _close(got, want)
    assert torch.equal(refreshed, cur)
    # the built-in array holds 16 samples: 17 is refused before any launch
    big = _abi.sol_residual_change_noalloc(cur.data_ptr(), prev.data_ptr(), None, 17, 1, 2048,
                                           ctypes.c_void_p(16).value, _abi.SOL_BF16, None)
    assert big == _abi.SOL_ERR_UNSUPPORTED
    assert "16 samples" in _abi.last_error()
