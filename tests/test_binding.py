"""The Python binding's own argument checks, on the CPU: they run before any CUDA call, so
a wrong tensor (host memory where device memory is expected, a wrong dtype or shape)
raises ValueError without touching a GPU and without a silent fallback."""
import pytest
import torch

import exact_attention_101_b200 as fa


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_device_entry_points_reject_host_tensors():
    q, k, v = bf16(1, 2, 64, 128), bf16(1, 2, 64, 128), bf16(1, 2, 64, 128)
    with pytest.raises(ValueError, match="CUDA"):
        fa.forward(q, k, v)
    with pytest.raises(ValueError, match="CUDA"):
        fa.forward_dropout(q, k, v, 0.1, seed=1)
    with pytest.raises(ValueError, match="CUDA"):
        fa.backward(q, k, v, q, torch.zeros(1, 2, 64), q)


def test_forward_host_checks_dtype_layout_and_shapes():
    q, k, v = bf16(1, 4, 64, 128), bf16(1, 2, 64, 128), bf16(1, 2, 64, 128)
    with pytest.raises(ValueError, match="bf16 host tensor"):
        fa.forward_host(q.float(), k, v)
    with pytest.raises(ValueError, match="bf16 host tensor"):
        fa.forward_host(q.transpose(1, 2), k, v)
    with pytest.raises(ValueError, match="bf16 host tensor"):
        fa.forward_host(q[0], k, v)
    with pytest.raises(ValueError, match="shapes"):
        fa.forward_host(q, k, bf16(1, 2, 65, 128))
    with pytest.raises(ValueError, match="shapes"):
        fa.forward_host(q, bf16(2, 2, 64, 128), bf16(2, 2, 64, 128))
    with pytest.raises(ValueError, match="out_dtype"):
        fa.forward_host(q, k, v, out_dtype=torch.float16)


def test_library_symbols_match_the_binding():
    """Every C entry point has a raw mirror of the same name in the binding."""
    for name in fa.C_SYMBOLS:
        assert callable(getattr(fa, name)), name
