"""The allocation-free change detector, sol_residual_change_noalloc.

It serves callers that cannot call cudaMalloc: hosts whose device memory
already belongs to their own pool or framework allocator, hot loops that
must not pay cudaMalloc's implicit synchronisation, plain-C plug-ins with no
allocator at hand.  It keeps its partial sums in an array inside libsol
instead of a caller workspace.

The entry point runs the same two kernels as sol_residual_change, in the same
fixed summation order, so its results must equal the workspace entry point's
bit for bit.  This test calls it through the C ABI twice in a row, on two
different inputs, and checks each result for that equality and, directly,
against the fp64 oracle within the tolerance the parity tests use (relative
1e-5).  A 16-sample call reaches the array's last sample block.  The inputs and outputs
here are allocated by the test; the entry point itself allocates nothing.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from video_diffusion_transformer_rms_b200 import _abi
from video_diffusion_transformer_rms_b200.workloads import to_oracle_array

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


def _oracle_close(got, cur, prev):
    """Relative error <= 1e-5 against the fp64 oracle (fp32 row partials of at
    most 64 terms, fp64 beyond)."""
    B, L, D = cur.shape
    want = oracle.residual_change(to_oracle_array(cur.reshape(-1, D)),
                                  to_oracle_array(prev.reshape(-1, D)), B, L)
    np.testing.assert_allclose(got.cpu().numpy(), want, rtol=1e-5, atol=1e-30)


def test_no_alloc_matches_workspace_entry_point_twice_in_a_row():
    assert torch.cuda.is_available(), "this test needs a CUDA device"
    _abi.lib()
    cases = [_inputs(2, 4099, 5120, seed=1), _inputs(3, 1500, 3072, seed=2)]
    wants = [_with_workspace(c, p) for c, p in cases]
    gots = [_no_alloc(c, p) for c, p in cases]  # two calls in a row
    torch.cuda.synchronize()
    for (cur, prev), got, want in zip(cases, gots, wants):
        assert torch.equal(got, want)
        _oracle_close(got, cur, prev)
        assert 0.0 < float(want[-1, 2]) < 1.0


def test_no_alloc_sixteen_samples_fill_the_array():
    # B = 16 is the largest batch the built-in array holds: the slots of
    # every sample, the array's last sample block included, are written and
    # read back
    cases = [_inputs(16, 257, 1024, seed=4), _inputs(16, 33, 5120, seed=5)]
    for cur, prev in cases:
        got = _no_alloc(cur, prev)
        want = _with_workspace(cur, prev)
        torch.cuda.synchronize()
        assert torch.equal(got, want)
        _oracle_close(got, cur, prev)


def test_no_alloc_cache_refresh_and_limit():
    cur, prev = _inputs(1, 777, 2048, seed=3)
    want = _with_workspace(cur, prev)
    refreshed = torch.empty_like(prev)
    got = _no_alloc(cur, prev, prev_out=refreshed)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    assert torch.equal(refreshed, cur)
    # the built-in array holds 16 samples: 17 is refused before any launch
    big = _abi.sol_residual_change_noalloc(cur.data_ptr(), prev.data_ptr(), None, 17, 1, 2048,
                                           ctypes.c_void_p(16).value, _abi.SOL_BF16, None)
    assert big == _abi.SOL_ERR_UNSUPPORTED
    assert "16 samples" in _abi.last_error()
