"""The Python binding rejects wrong arguments before anything reaches the library:
wrong dtype, host tensors, non-contiguous views and mismatched FP8 shapes. (No GPU
needed: these checks run on the host.)"""
import pytest
import torch

from diffusion_transformer_video_b200 import dit3d


def test_bf16_arguments_must_be_contiguous_device_bf16():
    x = torch.zeros(8, 16, dtype=torch.bfloat16)               # host tensor
    with pytest.raises(TypeError):
        dit3d.dit_gated_residual(x, x, x[:1], 8)
    with pytest.raises(TypeError):
        dit3d.dit_linear(torch.zeros(8, 16), torch.zeros(8, 16))  # fp32
    with pytest.raises(TypeError):
        dit3d.dit_adaln_modulate(torch.zeros(16, 8, dtype=torch.bfloat16).t(), x[:1], x[:1], 8)


def test_fp8_arguments_are_uint8_codes_of_matching_shapes():
    with pytest.raises(TypeError):
        dit3d.dit_quantize_e4m3(torch.zeros(16), 1.0)
    with pytest.raises(TypeError):
        dit3d.dit_attn_fwd_fp8(torch.zeros(4, 1, 128), torch.zeros(4, 1, 128),
                               torch.zeros(4, 1, 128), 1.0, 1.0, 1.0)
    with pytest.raises(TypeError):
        dit3d.dit_linear_fp8(torch.zeros(4, 16, dtype=torch.uint8), torch.zeros(4, 16, dtype=torch.uint8),
                             1.0, 1.0)   # host codes


def test_euler_step_rejects_host_tensors():
    x = torch.zeros(8, 16, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        dit3d.dit_flow_euler_step(x, x, torch.zeros(2), 4)
