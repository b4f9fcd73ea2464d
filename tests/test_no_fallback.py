"""The product path has no CPU or PyTorch fallback: without the CUDA library, or
with tensors that are not on a CUDA device, every call fails loudly."""
import pytest
import torch

import lm_head_linear_tmem_b200 as flce
from lm_head_linear_tmem_b200 import _native, build


def test_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(_native, "_lib", None)
    monkeypatch.setattr(build, "SO_PATH", str(tmp_path / "absent" / "_flce.so"))
    with pytest.raises(RuntimeError, match="not found"):
        _native.load(build_if_missing=False)


def test_failed_build_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(_native, "_lib", None)
    monkeypatch.setattr(build, "SO_PATH", str(tmp_path / "_flce.so"))
    monkeypatch.setenv("NVCC", str(tmp_path / "no-such-nvcc"))
    monkeypatch.setattr(build.shutil, "which", lambda name: None)
    monkeypatch.setattr(build.os.path, "exists",
                        lambda p: False if p.endswith(("nvcc", "_flce.so")) else True)
    with pytest.raises(RuntimeError):
        _native.load()


def test_host_tensors_are_rejected():
    h = torch.zeros(4, 64, dtype=torch.bfloat16)
    w = torch.zeros(16, 64, dtype=torch.bfloat16)
    y = torch.zeros(4, dtype=torch.int64)
    with pytest.raises(ValueError, match="CUDA"):
        flce.forward(h, w, y)
    with pytest.raises(ValueError, match="CUDA"):
        flce.backward(h, w, y, torch.zeros(4))
