"""Fused per-token hot path of a joint video+audio diffusion-transformer
block on NVIDIA B200 (sm_100a): RMS-AdaLN, the AdaLN-gated residual and
per-head QKNorm + 3D multimodal RoPE, as CUDA kernels behind a C ABI
(include/sol.h, libsol.so).

    from video_diffusion_transformer_rms_b200 import api
    y = api.rms_adaln(x, scale, shift, n_video)

The CUDA library is loaded on first use and must be built; there is no CPU
path.
"""
from ._abi import (SOL_BF16, SOL_F32, SolError, sol_gate_residual,  # noqa: F401
                   sol_gate_residual_rms_adaln, sol_last_error, sol_qknorm_rope3d,
                   sol_qknorm_rope3d_ex, sol_qknorm_rope3d_ex_tab, sol_qknorm_rope3d_tab,
                   sol_rope_table_build, sol_rope_table_bytes,
                   sol_residual_change, sol_residual_change_workspace_bytes,
                   sol_rms_adaln, sol_status_string, sol_version)

__version__ = "1.0"
