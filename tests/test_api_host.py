"""The tensor wrappers check what the C ABI cannot see (shapes, contiguity,
devices) before any pointer is passed.  CPU tensors are enough here: the shape
checks run before the CUDA-tensor check."""
import pytest
import torch

from video_diffusion_transformer_rms_b200 import api

Z = torch.zeros


def test_rms_adaln_checks_modulation_gamma_and_out():
    x = Z(2, 4, 16)
    with pytest.raises(ValueError, match="scale"):
        api.rms_adaln(x, Z(2, 16), Z(2, 2, 16), 2)          # scale missing its modality axis
    with pytest.raises(ValueError, match="shift"):
        api.rms_adaln(x, Z(2, 2, 16), Z(1, 2, 16), 2)       # shift for one sample only
    with pytest.raises(ValueError, match="gamma"):
        api.rms_adaln(x, Z(2, 2, 16), Z(2, 2, 16), 2, gamma=Z(8))
    with pytest.raises(ValueError, match="out"):
        api.rms_adaln(x, Z(2, 2, 16), Z(2, 2, 16), 2, out=Z(2, 16, 4).transpose(1, 2))
    with pytest.raises(ValueError, match="CUDA"):
        api.rms_adaln(x, Z(2, 2, 16), Z(2, 2, 16), 2)       # shapes fine: now the device


def test_gate_residual_and_fused_check_every_operand():
    h = Z(1, 4, 16)
    with pytest.raises(ValueError, match="branch"):
        api.gate_residual(h, Z(1, 16, 4).transpose(1, 2), Z(1, 2, 16), 2)  # strided branch
    with pytest.raises(ValueError, match="gate"):
        api.gate_residual(h, Z(1, 4, 16), Z(1, 16), 2)
    with pytest.raises(ValueError, match="y"):
        api.gate_residual_rms_adaln(h, Z(1, 4, 16), Z(1, 2, 16), Z(1, 2, 16), Z(1, 2, 16), 2,
                                    y=Z(1, 4, 8))


def test_residual_change_checks_prev_and_out():
    cur = Z(2, 4, 16)
    with pytest.raises(ValueError, match="prev"):
        api.residual_change(cur, Z(2, 4, 8))
    with pytest.raises(ValueError, match="out"):
        api.residual_change(cur, Z(2, 4, 16), out=Z(2, 3, dtype=torch.float64))
    with pytest.raises(TypeError, match="float64"):
        api.residual_change(cur, Z(2, 4, 16), out=Z(3, 3))


def test_qk_and_gemm_check_gamma_outputs_and_operands():
    qkv = Z(1, 56, 3 * 256)
    with pytest.raises(ValueError, match="gamma_q"):
        api.qknorm_rope3d(qkv, 2, 4, 6, 8, 2, 128, gamma_q=Z(64))
    with pytest.raises(ValueError, match="k_out"):
        api.qknorm_rope3d(qkv, 2, 4, 6, 8, 2, 128, q_out=Z(1, 56, 256), k_out=Z(1, 28, 256))
    with pytest.raises(ValueError, match="gamma_k"):
        api.qknorm_rope3d_ex(qkv, 2, 4, 6, 8, 2, 128, gamma_k=Z(2, 128))
    with pytest.raises(ValueError, match="bias"):
        api.gemm_gelu(Z(4, 8, dtype=torch.bfloat16), Z(16, 8, dtype=torch.bfloat16),
                      Z(8, dtype=torch.bfloat16))
