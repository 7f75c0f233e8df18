"""Helpers for comparing the CUDA path with the fp64 oracle (tests only)."""
import numpy as np
import torch

import oracle
from video_diffusion_transformer_rms_b200.workloads import to_oracle_array


def oracle_dtype(t: torch.Tensor) -> int:
    return oracle.F32 if t.dtype == torch.float32 else oracle.BF16


def gpu_values(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(got: torch.Tensor, want: np.ndarray, what: str):
    """|got - want| <= 2 ulp(want) + 1e-3 element by element (ulp of the I/O
    dtype at the oracle value), finite everywhere."""
    g = gpu_values(got).reshape(want.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    err = np.abs(g - want)
    tol = oracle.tolerance(want, oracle_dtype(got))
    bad = err > tol
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {err.size} elements out of tolerance; worst at "
            f"{i}: gpu={g[i]!r} oracle={want[i]!r} err={err[i]:.3e} tol={tol[i]:.3e}")
    return float(err.max()) if err.size else 0.0


def sample_rows(rows: int, L: int, n_video: int, B: int, n: int, seed: int) -> np.ndarray:
    """A seeded sample of global row ids that always includes every sample's
    first and last rows and both sides of its video/audio boundary."""
    rng = np.random.default_rng(seed)
    must = []
    for b in range(B):
        base = b * L
        for r in (0, 1, n_video - 1, n_video, n_video + 1, L - 2, L - 1):
            if 0 <= r < L:
                must.append(base + r)
    extra = rng.choice(rows, size=min(n, rows), replace=False)
    return np.unique(np.concatenate([np.array(must, dtype=np.int64), extra.astype(np.int64)]))


def take_rows(t: torch.Tensor, ids: np.ndarray) -> np.ndarray:
    """Exact host copy (oracle format) of the given rows of a [rows, C] tensor."""
    idx = torch.as_tensor(ids, device=t.device)
    return to_oracle_array(t.index_select(0, idx))


def take_rows_gpu(t: torch.Tensor, ids: np.ndarray) -> torch.Tensor:
    return t.index_select(0, torch.as_tensor(ids, device=t.device))
