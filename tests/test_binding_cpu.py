"""Host-side argument checks of the Python binding that need no GPU: the layer
classes' device normalisation and their input validation (a CPU tensor, a wrong
dtype, width or device is refused before anything reaches the C ABI)."""
import pytest
import torch

import diffusion_transformer_w4a4_b200 as svdq


def test_layer_device_keeps_an_explicit_index():
    assert svdq._layer_device("cuda:1") == torch.device("cuda", 1)
    assert svdq._layer_device(torch.device("cuda", 3)).index == 3


def test_layer_device_refuses_the_cpu():
    with pytest.raises(ValueError):
        svdq._layer_device("cpu")


def test_input_checks():
    dev = torch.device("cuda", 0)
    with pytest.raises(ValueError, match="CUDA tensor"):
        svdq._check_input(torch.zeros(4, 64, dtype=torch.bfloat16), 64, dev)  # on the CPU
    with pytest.raises(ValueError, match="CUDA tensor"):
        svdq._check_input(torch.zeros(4, 64, dtype=torch.float32), 64, dev)  # wrong dtype (checked first)
    with pytest.raises(ValueError, match="CUDA tensor"):
        svdq._check_input(torch.zeros(4, 32, dtype=torch.bfloat16), 64, dev)  # wrong width
