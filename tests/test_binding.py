"""The Python binding refuses tensors the C ABI cannot take, before any
pointer is passed on (no GPU needed: the checks run on the host)."""

import pytest
import torch

import quantized_fp8_attention_b200 as fqa


def _bf16(*shape, device="cpu"):
    return torch.zeros(*shape, dtype=torch.bfloat16, device=device)


def test_host_tensors_are_refused():
    q = _bf16(1, 1, 128, 128)
    with pytest.raises(ValueError, match="CUDA"):
        fqa.quantize(q, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        fqa.attention_bf16(q, q, q, fqa.softmax_scale())
    with pytest.raises(ValueError, match="CUDA"):
        fqa.e4m3_encode(torch.zeros(4))


def test_wrong_rank_and_type_are_refused():
    with pytest.raises(ValueError, match="B, H, N, 128"):
        fqa.quantize(_bf16(128, 128), _bf16(128, 128), _bf16(128, 128))
    with pytest.raises(TypeError):
        fqa._require([1, 2], torch.float32, "x")


def test_quantized_bundle_is_checked_field_by_field():
    # CPU tensors fail the device check of the first field
    qz = fqa.Quantized(*(torch.zeros(1) for _ in fqa.Quantized._fields))
    with pytest.raises(ValueError):
        fqa._require_quantized(qz, 1, 1, 128)
