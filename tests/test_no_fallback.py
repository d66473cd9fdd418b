"""The product path has no CPU or PyTorch fallback: without the CUDA library every call
raises, and host tensors are refused instead of being computed on."""
import pytest
import torch

from long_context_04_b200 import api


def test_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setenv("LA_LIBRARY", str(tmp_path / "absent.so"))
    monkeypatch.setattr(api, "_LIB", None)
    with pytest.raises(api.LightningLibraryError):
        api.lib()
    with pytest.raises(api.LightningLibraryError):
        api.version()
    with pytest.raises(api.LightningLibraryError):
        api.device_status()


def test_host_tensors_are_refused():
    q = torch.zeros(8, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        api.prefill(q, q, q, beta=64)
    with pytest.raises(ValueError, match="CUDA tensor"):
        api.decode_step(q, q, q, torch.zeros(8, 2, 64, 64))
    with pytest.raises(ValueError, match="CUDA tensor"):
        api.chunk_state(q, q)
