"""Seeded synthetic workloads for the per-token DiT hot path.

This module only draws random numbers and fixes shapes; it holds none of the
normalisation, modulation or rotary arithmetic.  Both the CUDA path and the
CPU oracle are fed from it (the oracle receives the exact device bits).

Shapes follow the joint video+audio sequence of a MiniMax-H3 style
single-stream DiT (ThakiCloud MiniMax-H3 post, spec table: 1344x768, 24 fps,
4-15 s clips; H3-OnDevice page: 124 frames at 1344x768): per sample, the
T*H*W video latent patches in raster order (t-major), then the audio tokens.

Distributions (one reading of "x~N(0,1)", "scale/shift~N(0,0.5)",
"gate~N(0,0.1)", "gamma~1+N(0,0.1)": the second number is the standard
deviation):
  x, h, branch, qkv : N(0, 1), with round(1% of the columns) chosen by the
                      seed and multiplied by 20 (outlier channels; the same
                      columns in every row); no outliers in the tiny case
  scale, shift      : N(0, 0.5), one [D] vector per (sample, modality)
  gate              : N(0, 0.1), one [D] vector per (sample, modality)
  gamma_q, gamma_k  : 1 + N(0, 0.1), [head_dim]
  gamma (optional RMS-AdaLN weight, not in the pages' configs): 1 + N(0, 0.1)
Values are drawn in fp32 and rounded once to the I/O dtype.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int            # position in the workload list; seeds derive from it
    B: int
    n_heads: int
    head_dim: int
    T: int
    H: int
    W: int
    n_audio: int
    dtype: str            # "f32" or "bf16"
    outliers: bool
    sections: tuple = (16, 24, 24)
    eps: float = 1e-6
    theta: float = 10000.0

    @property
    def D(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def n_video(self) -> int:
        return self.T * self.H * self.W

    @property
    def L(self) -> int:
        return self.n_video + self.n_audio

    @property
    def rows(self) -> int:
        return self.B * self.L

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def esize(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def bytes_per_row(self) -> Dict[str, int]:
        """Algorithmic HBM bytes per token row for each kernel."""
        e = self.esize
        return {
            "rms_adaln": 2 * self.D * e,        # read x, write y
            "gate_residual": 3 * self.D * e,    # read h, branch; write out
            "qknorm_rope3d": 4 * self.D * e,    # read q, k; write q, k
        }


# The five workload shapes (the last one repeated at D=3072).
WORKLOADS = {
    w.name: w for w in [
        # tiny oracle sanity check, fp32 I/O: 48 video + 8 audio rows
        Workload("tiny", 0, B=1, n_heads=2, head_dim=128, T=2, H=4, W=6,
                 n_audio=8, dtype="f32", outliers=False),
        # medium: 8x24x42 latent grid + 200 audio rows
        Workload("medium", 1, B=1, n_heads=40, head_dim=128, T=8, H=24, W=42,
                 n_audio=200, dtype="bf16", outliers=True),
        # 5 s 1344x768 24 fps clip: T=31 (124 frames / 4), H=768/16, W=1344/16
        Workload("clip5s", 2, B=1, n_heads=40, head_dim=128, T=31, H=48, W=84,
                 n_audio=1560, dtype="bf16", outliers=True),
        # 15 s clip: T=91
        Workload("clip15s", 3, B=1, n_heads=40, head_dim=128, T=91, H=48, W=84,
                 n_audio=4680, dtype="bf16", outliers=True),
        # classifier-free-guidance batch at the 5 s shape, two samples
        Workload("cfg5s", 4, B=2, n_heads=40, head_dim=128, T=31, H=48, W=84,
                 n_audio=1560, dtype="bf16", outliers=True),
        # the same at hidden size 3072 (24 heads)
        Workload("cfg5s_d3072", 4, B=2, n_heads=24, head_dim=128, T=31, H=48,
                 W=84, n_audio=1560, dtype="bf16", outliers=True),
    ]
}

# tensor ids for the seeds: seed = 1000 * workload.index + id (+100 for D=3072)
_TENSOR_IDS = {"x": 1, "scale": 2, "shift": 3, "gate": 4, "h": 5, "branch": 6,
               "qkv": 7, "gamma_q": 8, "gamma_k": 9, "gamma": 10}


def seed_for(w: Workload, tensor: str) -> int:
    extra = 100 if w.name.endswith("_d3072") else 0
    return 1000 * w.index + _TENSOR_IDS[tensor] + extra


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def outlier_columns(width: int, seed: int, device="cpu") -> torch.Tensor:
    """round(1% of width) distinct columns, chosen by the seed."""
    n = int(round(0.01 * width))
    g = _gen("cpu", seed + 500_000)
    cols = torch.randperm(width, generator=g)[:n]
    return torch.sort(cols).values.to(device)


def activation(rows: int, width: int, dtype: torch.dtype, device, seed: int,
               outliers: bool, chunk_rows: int = 8192,
               out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """[rows, width] ~ N(0,1) with the seeded outlier columns scaled by 20.

    Drawn in row chunks so that a 15 s clip's QKV (5.7e9 elements) never
    needs an fp32 copy of the whole tensor.
    """
    if out is None:
        out = torch.empty((rows, width), dtype=dtype, device=device)
    g = _gen(device, seed)
    cols = outlier_columns(width, seed, device) if outliers else None
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        blk = torch.randn((r1 - r0, width), generator=g, device=device,
                          dtype=torch.float32)
        if cols is not None and cols.numel():
            blk[:, cols] *= 20.0
        out[r0:r1].copy_(blk)
    return out


def vectors(shape, mean: float, std: float, dtype, device, seed: int) -> torch.Tensor:
    g = _gen(device, seed)
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return (v * std + mean).to(dtype)


def make_inputs(w: Workload, device="cpu", which=("rms_adaln", "gate_residual",
                                                  "qknorm_rope3d"),
                with_gamma: bool = False) -> Dict[str, torch.Tensor]:
    """All inputs a workload needs, on `device`, in the workload's I/O dtype."""
    dt = w.torch_dtype
    t: Dict[str, torch.Tensor] = {}
    if "rms_adaln" in which:
        t["x"] = activation(w.rows, w.D, dt, device, seed_for(w, "x"), w.outliers)
        t["scale"] = vectors((w.B, 2, w.D), 0.0, 0.5, dt, device, seed_for(w, "scale"))
        t["shift"] = vectors((w.B, 2, w.D), 0.0, 0.5, dt, device, seed_for(w, "shift"))
        if with_gamma:
            t["gamma"] = vectors((w.D,), 1.0, 0.1, dt, device, seed_for(w, "gamma"))
    if "gate_residual" in which:
        t["h"] = activation(w.rows, w.D, dt, device, seed_for(w, "h"), w.outliers)
        t["branch"] = activation(w.rows, w.D, dt, device, seed_for(w, "branch"), w.outliers)
        t["gate"] = vectors((w.B, 2, w.D), 0.0, 0.1, dt, device, seed_for(w, "gate"))
    if "qknorm_rope3d" in which:
        t["qkv"] = activation(w.rows, 3 * w.D, dt, device, seed_for(w, "qkv"), w.outliers)
        t["gamma_q"] = vectors((w.head_dim,), 1.0, 0.1, dt, device, seed_for(w, "gamma_q"))
        t["gamma_k"] = vectors((w.head_dim,), 1.0, 0.1, dt, device, seed_for(w, "gamma_k"))
    return t


def to_oracle_array(t: torch.Tensor):
    """Exact host copy of a tensor's bits for the oracle: float32 stays
    float32, bf16 becomes its uint16 bit pattern."""
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(f"unsupported dtype {t.dtype}")
